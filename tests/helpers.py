"""Shared helpers for the GPU parity tests: run the CUDA path and the CPU oracle on the
same seeded fp32 inputs and compare. Oracle inputs and expected values come only from the
seeded generators and from ``oracle``; nothing computed by the CUDA path feeds the oracle."""
from __future__ import annotations

import numpy as np
import torch

import nvfp4_block_scaled_08_b200 as nv
import oracle

TOL_REL = 2.0 ** -7


def gpu_quantize(x_cpu: torch.Tensor, dev, dtype=torch.float32):
    """CUDA path: global scale then quantisation of a CPU fp32 tensor copied to `dev`."""
    x = x_cpu.to(dtype).to(dev)
    gs = nv.global_scale(x)
    q, sf = nv.quantize(x, gs)
    return q, sf, gs


def oracle_quantize(x_cpu: torch.Tensor, dtype=torch.float32, gs=None):
    """Oracle: the same steps on the CPU (a bf16 input is widened to fp32 exactly first)."""
    x = x_cpu.to(dtype).to(torch.float32).numpy()
    if gs is None:
        gs = oracle.global_scale(x)
    q, sf = oracle.quantize(x, gs)
    return q, sf, gs


def check_within_tolerance(out_gpu: torch.Tensor, v: np.ndarray, S: np.ndarray, alpha, what=""):
    """|out - v| <= 2^-7 |alpha| S + 1e-6 per element (out is bf16 from the GPU)."""
    got = out_gpu.float().cpu().numpy().astype(np.float64)
    assert got.shape == v.shape, (got.shape, v.shape)
    tol = oracle.tolerance(S, alpha)
    err = np.abs(got - v)
    bad = err > tol
    if bad.any():
        idx = np.argwhere(bad)[:5]
        details = [(tuple(i), got[tuple(i)], v[tuple(i)], tol[tuple(i)]) for i in idx]
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance, e.g. {details}")
    assert np.isfinite(got).all()
    return float((err / np.maximum(tol, 1e-30)).max())


def bf16_bits_of(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def tile_np(sf: np.ndarray, K: int) -> np.ndarray:
    """The tiled layout: row r, scale column c at ((r // 128) * (K // 64) + c // 4) * 512
    + (r % 32) * 16 + ((r // 32) % 4) * 4 + c % 4; rows padded to 128 with zeros."""
    rows, kb = sf.shape
    assert kb == K // 16
    R = (rows + 127) // 128 * 128
    out = np.zeros(R * kb, dtype=np.uint8)
    r = np.arange(rows)[:, None]
    c = np.arange(kb)[None, :]
    off = ((r // 128) * (K // 64) + c // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + c % 4
    out[off] = sf
    return out


def layout_8x4_np(sf: np.ndarray, K: int) -> np.ndarray:
    """The 8 x 4 layout: row r, scale column c at ((r // 8) * (K // 64) + c // 4) * 32
    + (r % 8) * 4 + c % 4; rows padded to 8 with zeros."""
    rows, kb = sf.shape
    assert kb == K // 16
    R = (rows + 7) // 8 * 8
    out = np.zeros(R * kb, dtype=np.uint8)
    r = np.arange(rows)[:, None]
    c = np.arange(kb)[None, :]
    off = ((r // 8) * (K // 64) + c // 4) * 32 + (r % 8) * 4 + c % 4
    out[off] = sf
    return out
