"""The 8 x 4 scale layout (NVFP4_SF_8X4 in include/nvfp4.h) on the CPU.

The GPU tests compare the kernels with ``helpers.layout_8x4_np``, the layout's index formula
in NumPy. Here that formula is checked against the layout built block by block from its
definition: 32-byte blocks, each the scales of 8 consecutive rows for 4 consecutive scale
columns (64 K-elements), row-major inside the block; a row group's blocks follow one another
along K, then the next row group. The formula must also be a bijection onto the padded buffer
and keep a row group's four blocks of one 256-element K stage in one 128-byte run (the box the
GEMM's 2D copy fetches), with a stage's runs of consecutive row groups K / 2 bytes apart.
"""
import numpy as np
import pytest

from helpers import layout_8x4_np


def layout_by_blocks(sf: np.ndarray, K: int) -> np.ndarray:
    rows, kb = sf.shape
    R = (rows + 7) // 8 * 8
    padded = np.zeros((R, kb), np.uint8)
    padded[:rows] = sf
    out = []
    for g in range(R // 8):
        for j in range(kb // 4):
            out.append(padded[8 * g:8 * g + 8, 4 * j:4 * j + 4].reshape(-1))   # 8 rows x 4 bytes
    return np.concatenate(out)


@pytest.mark.parametrize("rows,K", [(1, 64), (7, 64), (8, 256), (9, 512), (37, 768), (300, 512), (64, 6144)])
def test_formula_matches_block_construction(rows, K):
    rng = np.random.default_rng(rows * 11 + K)
    sf = rng.integers(0, 256, (rows, K // 16), dtype=np.uint8)
    got = layout_8x4_np(sf, K)
    assert got.size == (rows + 7) // 8 * 8 * (K // 16)
    np.testing.assert_array_equal(got, layout_by_blocks(sf, K))


def test_formula_is_a_bijection_with_stage_runs():
    rows, K = 45, 1024
    kb = K // 16
    R = (rows + 7) // 8 * 8
    ids = np.arange(1, rows * kb + 1, dtype=np.int64).reshape(rows, kb)    # 0 marks padding
    where = sum(layout_8x4_np(((ids >> (8 * k)) & 0xFF).astype(np.uint8), K).astype(np.int64) << (8 * k)
                for k in range(3))
    assert where.size == R * kb
    placed = where[where > 0]
    assert placed.size == rows * kb and np.unique(placed).size == rows * kb
    # row group g, K stage s: bytes [g * K/2 + 128 s, + 128) hold rows 8g..8g+7, columns
    # 16 s .. 16 s + 15, k-step j's four columns of row r at 32 j + 4 (r % 8)
    for g in range(R // 8):
        for s in range(kb // 16):
            run = where[g * (K // 2) + 128 * s:g * (K // 2) + 128 * s + 128]
            for r in range(8 * g, min(8 * g + 8, rows)):
                for j in range(4):
                    w = run[32 * j + 4 * (r % 8):32 * j + 4 * (r % 8) + 4]
                    np.testing.assert_array_equal(w, ids[r, 16 * s + 4 * j:16 * s + 4 * j + 4])
