"""Pins for the oracle's MXFP4 functions (the use_nvfp4=False variant of the mm_fp4 signature
in "The Art of Reading the Manual", section "The Message"; format: OCP MX v1.0 FP4, e2m1
elements with one E8M0 power-of-two scale per 32 elements). Each check compares the oracle
with something other than itself:

* E8M0 values: ml_dtypes' and torch's float8_e8m0fnu.
* Scale exponents: a brute-force search for the largest power of two 2^s with
  4 * 2^s <= amax, clamped to the E8M0 range, plus closed forms at the binade edges.
* Codes: ml_dtypes' float4_e2m1fn conversion of x / 2^s.
* Reconstruction: the e2m1 half-step bound, or the clipping error above 6 * 2^s.
* Products: exact rational arithmetic (fractions.Fraction) on operands decoded by ml_dtypes,
  transposition, linearity in alpha, and the exactness flag on a wide exponent span.
"""
import math
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

F4 = ml_dtypes.float4_e2m1fn
E8 = ml_dtypes.float8_e8m0fnu


def blocks(x):
    rows, K = x.shape
    return x.reshape(rows, K // 32, 32)


def lib_codes(q):
    """Codes of q as values, decoded by ml_dtypes (low nibble first)."""
    lo = (q & 0xF).view(F4).astype(np.float64)
    hi = (q >> 4).view(F4).astype(np.float64)
    return np.stack([lo, hi], axis=-1).reshape(q.shape[0], q.shape[1] * 2)


def brute_shared_exp(amax: float) -> int:
    if amax == 0.0:
        return -127
    best = -127
    for s in range(-127, 128):
        if 4.0 * 2.0 ** s <= amax:      # 2^(s+2) <= amax: floor(log2(amax)) >= s + 2
            best = s
    return best


def test_e8m0_table_matches_libraries():
    lib = np.arange(256, dtype=np.uint8).view(E8).astype(np.float64)
    tor = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    for b in range(256):
        v = oracle.e8m0_decode(b)
        if b == 255:
            assert math.isnan(v) and math.isnan(lib[b]) and math.isnan(tor[b])
        else:
            assert v == lib[b] == tor[b] == 2.0 ** (b - 127), b


def _inputs(seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((6, 128)).astype(np.float32)
    x[1] *= np.float32(2.0 ** 40)                         # large and small binades
    x[2] *= np.float32(2.0 ** -60)
    x[3, :32] = 0.0                                       # a zero block
    x[3, 32:64] = np.float32(-2.5)                        # a constant negative block
    x[4] = rng.uniform(-1, 1, 128).astype(np.float32) * np.exp2(rng.integers(-20, 20, 128)).astype(np.float32)
    x[5, :32] = np.float32(2.0 ** -140)                   # subnormal block
    return x


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_scale_bytes_brute_force(seed):
    x = _inputs(seed)
    _, sf = oracle.mx_quantize(x)
    amax = np.abs(blocks(x)).max(axis=-1)
    for r in range(x.shape[0]):
        for b in range(x.shape[1] // 32):
            assert sf[r, b] == brute_shared_exp(float(amax[r, b])) + 127, (r, b, amax[r, b])


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_codes_match_library_conversion(seed):
    x = _inputs(seed)
    q, sf = oracle.mx_quantize(x)
    scale = np.repeat(sf.astype(np.int64) - 127, 32, axis=1)
    y = np.ldexp(x.astype(np.float64), -scale).astype(np.float32)    # exact quotient
    ref = y.astype(F4).view(np.uint8)
    ours = np.stack([q & 0xF, q >> 4], axis=-1).reshape(x.shape)
    np.testing.assert_array_equal(ours, ref)


@pytest.mark.parametrize("k", [-100, -3, 0, 5, 90])
def test_closed_forms_at_binade_edges(k):
    x = np.zeros((4, 32), np.float32)
    x[0, 0] = np.float32(6.0 * 2.0 ** k)     # largest element exactly representable: code 7
    x[1, 0] = np.float32(4.0 * 2.0 ** k)     # 2^(k+2): scale 2^k, value 4 (code 6)
    x[2, 0] = np.float32(7.9 * 2.0 ** k)     # scale 2^k, clipped to 6 (code 7)
    x[3, 0] = np.float32(8.0 * 2.0 ** k)     # next binade: scale 2^(k+1), value 4 (code 6)
    x[:, 1] = np.float32(-0.0)
    q, sf = oracle.mx_quantize(x)
    assert sf[:, 0].tolist() == [127 + k, 127 + k, 127 + k, 128 + k]
    assert [int(q[r, 0] & 0xF) for r in range(4)] == [7, 6, 7, 6]
    assert all(int(q[r, 0] >> 4) == 8 for r in range(4))           # -0.0 keeps its sign
    assert (q[:, 1:] == 0).all()


def test_zero_block_and_sign_symmetry():
    x = np.zeros((2, 64), np.float32)
    x[0, 32:] = np.linspace(-3, 3, 32, dtype=np.float32)
    q, sf = oracle.mx_quantize(x)
    assert sf[0, 0] == 0 and sf[1].tolist() == [0, 0] and (q[1] == 0).all()
    qn, sfn = oracle.mx_quantize(-x)
    np.testing.assert_array_equal(sfn, sf)
    codes = np.stack([q & 0xF, q >> 4], axis=-1).reshape(2, 64)
    codes_n = np.stack([qn & 0xF, qn >> 4], axis=-1).reshape(2, 64)
    np.testing.assert_array_equal(codes_n ^ 8, codes)


@pytest.mark.parametrize("seed", [3, 4])
def test_reconstruction_bound(seed):
    x = _inputs(seed)
    q, sf = oracle.mx_quantize(x)
    deq = oracle.mx_dequantize(q, sf)
    X = np.repeat(np.ldexp(1.0, sf.astype(np.int64) - 127), 32, axis=1)
    np.testing.assert_array_equal(deq, lib_codes(q) * X)
    y = np.abs(x.astype(np.float64)) / X
    assert (y < 8.0).all()                                 # floor(log2 amax) - 2 keeps |y| < 8
    half_step = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0))
    bound = np.maximum(half_step, y - 6.0) * X
    assert (np.abs(deq - x) <= bound * (1 + 1e-12)).all()


def _exact_product(deqA, deqB, alpha):
    M, K = deqA.shape
    N = deqB.shape[0]
    out = np.empty((M, N))
    for m in range(M):
        for n in range(N):
            acc = sum((Fraction(float(deqA[m, k])) * Fraction(float(deqB[n, k])) for k in range(K)),
                      Fraction(0))
            out[m, n] = float(Fraction(float(np.float32(alpha))) * acc)
    return out


@pytest.mark.parametrize("M,N,K,seed", [(3, 4, 64, 5), (5, 3, 96, 6)])
def test_gemm_exact_rationals(M, N, K, seed):
    rng = np.random.default_rng(seed)
    a = (rng.standard_normal((M, K)) * np.exp2(rng.integers(-8, 8, (M, 1)))).astype(np.float32)
    b = (rng.standard_normal((N, K)) * np.exp2(rng.integers(-8, 8, (N, 1)))).astype(np.float32)
    qa, sa = oracle.mx_quantize(a)
    qb, sb = oracle.mx_quantize(b)
    alpha = 0.37
    v, S, exact = oracle.mx_gemm(qa, sa, qb, sb, alpha, threads=2)
    assert exact
    deqA = lib_codes(qa) * np.repeat(np.ldexp(1.0, sa.astype(np.int64) - 127), 32, axis=1)
    deqB = lib_codes(qb) * np.repeat(np.ldexp(1.0, sb.astype(np.int64) - 127), 32, axis=1)
    np.testing.assert_array_equal(v, _exact_product(deqA, deqB, alpha))
    np.testing.assert_allclose(S, np.abs(deqA) @ np.abs(deqB).T, rtol=1e-15)


def test_gemm_transpose_alpha_and_zero():
    rng = np.random.default_rng(8)
    a = rng.standard_normal((7, 128)).astype(np.float32)
    b = rng.standard_normal((5, 128)).astype(np.float32)
    qa, sa = oracle.mx_quantize(a)
    qb, sb = oracle.mx_quantize(b)
    v, _, _ = oracle.mx_gemm(qa, sa, qb, sb, 1.0)
    vt, _, _ = oracle.mx_gemm(qb, sb, qa, sa, 1.0)
    np.testing.assert_array_equal(v, vt.T)
    v4, _, _ = oracle.mx_gemm(qa, sa, qb, sb, 4.0)
    np.testing.assert_array_equal(v4, 4.0 * v)
    z, Sz, _ = oracle.mx_gemm(np.zeros_like(qa), sa, qb, sb, 1.0)
    assert (z == 0).all() and (Sz == 0).all()


def test_exactness_flag_on_wide_exponent_span():
    # 2^30 + 2^-30 needs 61 significant bits, so no fp64 sum of the two products is exact and
    # the flag must say so; 2^30 + 2^-10 fits in 41 bits and is exact
    b = np.ones((1, 64), np.float32)
    qb, sb = oracle.mx_quantize(b)
    a = np.zeros((1, 64), np.float32)
    a[0, 0] = np.float32(2.0 ** 30)
    a[0, 32] = np.float32(2.0 ** -30)
    qa, sa = oracle.mx_quantize(a)
    v, _, exact = oracle.mx_gemm(qa, sa, qb, sb, 1.0)
    assert not exact and v[0, 0] == 2.0 ** 30
    a[0, 32] = np.float32(2.0 ** -10)
    qa, sa = oracle.mx_quantize(a)
    v, _, exact = oracle.mx_gemm(qa, sa, qb, sb, 1.0)
    assert exact and v[0, 0] == 2.0 ** 30 + 2.0 ** -10
