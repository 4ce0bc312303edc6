"""The tiled scale layout (NVFP4_SF_TILED in include/nvfp4.h) on the CPU.

The GPU tests compare the kernels with ``helpers.tile_np``, the layout's index formula in
NumPy. Here that formula is checked against a second derivation: the layout built block by
block from what it is for. Each 512-byte block is the source operand of one
``tcgen05.cp ... 32x128b.warpx4`` copy: 32 rows of 16 bytes, where row i holds four
consecutive scale columns of rows i, i + 32, i + 64 and i + 96 of a 128-row tile. Blocks run
along K within a row tile, then tile after tile. The formula must also be a bijection onto
the padded buffer and keep a row tile's four consecutive blocks in one 2 KB run.
"""
import numpy as np
import pytest

from helpers import tile_np


def tile_by_blocks(sf: np.ndarray, K: int) -> np.ndarray:
    rows, kb = sf.shape
    R = (rows + 127) // 128 * 128
    padded = np.zeros((R, kb), np.uint8)
    padded[:rows] = sf
    out = []
    for t in range(R // 128):
        for j in range(kb // 4):
            block = np.zeros((32, 16), np.uint8)
            for i in range(32):
                for s in range(4):
                    block[i, 4 * s:4 * s + 4] = padded[128 * t + 32 * s + i, 4 * j:4 * j + 4]
            out.append(block.reshape(-1))
    return np.concatenate(out)


@pytest.mark.parametrize("rows,K", [(1, 64), (32, 64), (128, 256), (129, 512), (300, 512), (256, 6144)])
def test_formula_matches_block_construction(rows, K):
    rng = np.random.default_rng(rows * 7 + K)
    sf = rng.integers(0, 256, (rows, K // 16), dtype=np.uint8)
    got = tile_np(sf, K)
    assert got.size == (rows + 127) // 128 * 128 * (K // 16)
    np.testing.assert_array_equal(got, tile_by_blocks(sf, K))


def test_formula_is_a_bijection_with_contiguous_stage_runs():
    rows, K = 300, 1024
    kb = K // 16
    R = (rows + 127) // 128 * 128
    ids = np.arange(1, rows * kb + 1, dtype=np.int64).reshape(rows, kb)    # 0 marks padding
    # which scale lands in each byte of the tiled buffer: tile the ids one byte plane at a time
    where = sum(tile_np(((ids >> (8 * k)) & 0xFF).astype(np.uint8), K).astype(np.int64) << (8 * k)
                for k in range(3))
    assert where.size == R * kb
    placed = where[where > 0]
    assert placed.size == rows * kb and np.unique(placed).size == rows * kb    # each scale once
    # a row tile's scale columns 16 s .. 16 s + 15 (one 256-element K step = four blocks) fill
    # exactly one 2 KB run, in the tile's K order
    for t in range(R // 128):
        for s in range(kb // 16):
            base = (t * (K // 64) + 4 * s) * 512
            run = where[base:base + 2048]
            want = ids[128 * t:min(128 * (t + 1), rows), 16 * s:16 * s + 16]
            assert np.array_equal(np.sort(run[run > 0]), np.sort(want.reshape(-1)))
