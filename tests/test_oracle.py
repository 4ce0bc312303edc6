"""Pins for the CPU oracle: each check compares it with something other than itself.

* Format tables and encoders: the ml_dtypes library (float4_e2m1fn, float8_e4m3fn),
  torch's float8_e4m3fn conversion, and brute-force nearest-value search.
* Quantisation: closed forms (the amax block gets scale 448 and code 6.0, constant blocks,
  constant tensors that dequantise back to themselves, zero blocks, sign symmetry, nibble
  order) and the NVFP4 reconstruction-error bound.
* Products: exact rational arithmetic (fractions.Fraction) on small random cases with the
  operand values decoded by ml_dtypes, all-zero scales, one-hot rows, transposition,
  linearity in alpha, and the grouped form against per-expert products.
* bf16 output rounding: brute-force nearest bf16 with ties to even; fp16 output
  rounding: numpy's conversion and a nearest-value search.
"""
import math
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

F4 = ml_dtypes.float4_e2m1fn
F8 = ml_dtypes.float8_e4m3fn


def lib_e2m1_values():
    return np.arange(16, dtype=np.uint8).view(F4).astype(np.float64)


def lib_e4m3_values():
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


# ---------------------------------------------------------------- format tables

def test_e2m1_table_matches_library():
    lib = lib_e2m1_values()
    for c in range(16):
        v = oracle.e2m1_decode(c)
        assert v == lib[c]
        assert math.copysign(1.0, v) == math.copysign(1.0, lib[c])
    # magnitudes of the 8 non-negative codes
    assert [oracle.e2m1_decode(c) for c in range(8)] == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_e4m3_table_matches_torch():
    lib = lib_e4m3_values()
    for b in range(256):
        v = oracle.e4m3_decode(b)
        if np.isnan(lib[b]):
            assert math.isnan(v), b
        else:
            assert v == lib[b], b
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0x38) == 1.0


# ---------------------------------------------------------------- encoders

def _midpoints_and_neighbours(values):
    vals = np.unique(np.abs(values[np.isfinite(values)]))
    mids = (vals[:-1] + vals[1:]) / 2.0
    pts = np.concatenate([vals, mids]).astype(np.float32)
    up = np.nextafter(pts, np.float32(np.inf))
    dn = np.nextafter(pts, np.float32(0))
    allp = np.concatenate([pts, up, dn])
    return np.concatenate([allp, -allp]).astype(np.float32)


def _random_floats(n, lo_exp, hi_exp, seed):
    rng = np.random.default_rng(seed)
    mant = rng.random(n) + 1.0
    exp = rng.integers(lo_exp, hi_exp, n)
    sign = rng.choice([-1.0, 1.0], n)
    return (sign * mant * np.exp2(exp)).astype(np.float32)


def test_e4m3_encode_matches_torch_below_saturation():
    x = np.concatenate([_midpoints_and_neighbours(lib_e4m3_values()),
                        _random_floats(200_000, -14, 9, 1),
                        np.array([0.0, -0.0, 2 ** -10, 2 ** -11, 1e-30, 1e-45], np.float32)])
    x = x[np.abs(x) < 464.0]          # torch maps >= 480-ish to NaN; saturation is tested below
    ours = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ref)
    ref2 = x.astype(F8).view(np.uint8)
    np.testing.assert_array_equal(ours, ref2)


def test_e4m3_encode_saturates_finite():
    x = np.array([448.0, 448.5, 463.9, 464.0, 479.0, 480.0, 1e6, 3.0e38], np.float32)
    assert (oracle.e4m3_encode(x) == 0x7E).all()
    assert (oracle.e4m3_encode(-x) == 0xFE).all()


def _nearest_even(values_by_code, y, n_codes):
    """Brute force: nearest magnitude; ties -> the code with mantissa bit 0."""
    a = abs(float(y))
    best, best_d = None, None
    for c in range(n_codes):
        d = abs(values_by_code[c] - a)
        if best is None or d < best_d or (d == best_d and c % 2 == 0 and best % 2 == 1):
            best, best_d = c, d
    return best


def test_e4m3_encode_brute_force():
    vals = [oracle.e4m3_decode(b) for b in range(0x7F)]   # 0x00..0x7E, non-negative finite
    rng = np.random.default_rng(7)
    x = np.concatenate([_random_floats(3000, -12, 9, 2), rng.random(1000).astype(np.float32) * 448,
                        _midpoints_and_neighbours(np.array(vals))])
    x = np.abs(x)
    x = x[x < 448.0]
    got = oracle.e4m3_encode(x)
    for xi, gi in zip(x, got):
        assert gi == _nearest_even(vals, xi, 0x7F), (xi, gi)


def test_e2m1_encode_matches_library_and_brute_force():
    table = lib_e2m1_values()
    x = np.concatenate([_midpoints_and_neighbours(table), _random_floats(200_000, -4, 4, 3),
                        np.array([0.0, -0.0, 7.0, -7.0, 1e30, -1e30, 1e-40, -1e-40], np.float32)])
    ours = oracle.e2m1_encode(x)
    np.testing.assert_array_equal(ours, x.astype(F4).view(np.uint8))
    mags = [abs(t) for t in table[:8]]
    for xi, oi in zip(x[:5000], ours[:5000]):
        c = _nearest_even(mags, xi, 8)
        sign = 8 if math.copysign(1.0, float(xi)) < 0 else 0
        assert oi == (c | sign), (xi, oi)


def test_e2m1_negative_zero_code():
    # Reading: the sign bit copies the input's sign, so tiny negatives give 0x8.
    assert oracle.e2m1_encode(np.array([-0.1, -0.0, 0.1], np.float32)).tolist() == [8, 8, 0]


# ---------------------------------------------------------------- quantisation

def test_global_scale_closed_forms():
    assert oracle.global_scale(np.zeros(64, np.float32)) == np.float32(1.0)
    assert oracle.global_scale(np.array([1.0, -6.0, 2.0], np.float32)) == np.float32(448.0)
    x = np.random.default_rng(0).standard_normal(4096).astype(np.float32)
    gs = oracle.global_scale(x)
    assert gs == np.float32(2688.0) / np.float32(np.abs(x).max())


def test_quantize_amax_block_gets_max_scale_and_code():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((8, 256)).astype(np.float32)
    gs = oracle.global_scale(x)
    q, sf = oracle.quantize(x, gs)
    r, k = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert sf[r, k // 16] == 0x7E
    code = (q[r, k // 2] >> (4 * (k % 2))) & 0xF
    assert code & 7 == 7
    assert (code >> 3) == (1 if x[r, k] < 0 else 0)
    # every other block scale is at most the maximum
    assert sf.max() == 0x7E


def test_quantize_constant_zero_and_sign():
    x = np.zeros((2, 64), np.float32)
    x[0, 16:32] = 0.37                       # a constant block
    x[0, 0:16] = 5.0                         # the tensor amax block
    gs = oracle.global_scale(x)
    q, sf = oracle.quantize(x, gs)
    codes = np.stack([q & 0xF, q >> 4], axis=-1).reshape(2, 64)
    assert (codes[0, 16:32] == 7).all()      # constant block -> all 6.0
    assert (codes[0, 0:16] == 7).all() and sf[0, 0] == 0x7E
    assert (codes[1] == 0).all() and (sf[1] == 0).all()     # zero rows
    qn, sfn = oracle.quantize(-x, gs)
    np.testing.assert_array_equal(sfn, sf)
    codes_n = np.stack([qn & 0xF, qn >> 4], axis=-1).reshape(2, 64)
    np.testing.assert_array_equal(codes_n, codes | 8)


@pytest.mark.parametrize("c", [1.0, 0.25, 1024.0, -8.0, 0.1, 3.7e-5, -12345.678, 448.0 * 6])
def test_constant_tensor_reproduces_itself(c):
    """A constant tensor: gs = 2688 / |c|, every block scale rounds to 448 (0x7E) and every
    code to 6.0, so the dequantised value over gs is 2688 / fl(2688 / |c|), within one fp32
    rounding of c, and exactly c when |c| is a power of two."""
    x = np.full((3, 48), c, np.float32)
    gs = oracle.global_scale(x)
    q, sf = oracle.quantize(x, gs)
    assert (sf == 0x7E).all()
    code = 7 | (8 if c < 0 else 0)
    assert (q == (code | code << 4)).all()
    back = oracle.dequantize(q, sf) / np.float64(gs)
    cf = np.float64(np.float32(c))
    assert np.all(np.abs(back - cf) <= 2.0 ** -23 * abs(cf))
    if math.frexp(abs(cf))[0] == 0.5:
        assert np.all(back == cf)


def test_quantize_nibble_order():
    # Reading: element 2i of a row goes in the low nibble of byte i.
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 1.0
    q, _ = oracle.quantize(x, oracle.global_scale(x))
    assert q[0, 0] == 0x07
    x = np.zeros((1, 16), np.float32)
    x[0, 1] = 1.0
    q, _ = oracle.quantize(x, oracle.global_scale(x))
    assert q[0, 0] == 0x70


def test_quantize_steps_match_library_conversions():
    """The same recipe evaluated with numpy fp32 arithmetic and ml_dtypes conversions."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((16, 512)) * np.exp2(rng.integers(-6, 6, (16, 1)))).astype(np.float32)
    x[3, 32:48] = 0.0
    gs = oracle.global_scale(x)
    q, sf = oracle.quantize(x, gs)
    blocks = x.reshape(16, 32, 16)
    amax = np.abs(blocks).max(-1)
    sf32 = (amax / np.float32(6.0)).astype(np.float32) * np.float32(gs)
    sf_lib = sf32.astype(np.float32).astype(F8)
    np.testing.assert_array_equal(sf, sf_lib.view(np.uint8))
    sfd = sf_lib.astype(np.float32)
    with np.errstate(divide="ignore"):
        rcp = np.where(sfd == 0, np.float32(0), np.float32(gs) / np.where(sfd == 0, 1, sfd))
    y = (blocks * rcp.astype(np.float32)[..., None]).astype(np.float32)
    codes = y.astype(F4).view(np.uint8).reshape(16, 512)
    np.testing.assert_array_equal(q, codes[:, 0::2] | (codes[:, 1::2] << 4))


def test_quantize_reconstruction_bound():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((32, 1024)).astype(np.float32)
    gs = oracle.global_scale(x)
    q, sf = oracle.quantize(x, gs)
    deq = oracle.dequantize(q, sf) / float(gs)
    sfd = lib_e4m3_values()[sf].repeat(16, axis=1)
    # e2m1 spacing is at most 2 (between 4 and 6): rounding error <= 1 unit of scale,
    # and saturation past 6 costs at most 6 * (1/16) units (e4m3 scale rounding).
    assert (np.abs(deq - x) <= sfd / float(gs) * 1.0 + 1e-12).all()


# ---------------------------------------------------------------- products

def _random_operands(rows, K, rng, scale_lo=0x20, scale_hi=0x48):
    q = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    sf = rng.integers(scale_lo, scale_hi, (rows, K // 16), dtype=np.uint8)
    return q, sf


def _lib_deq(q, sf):
    codes = np.stack([q & 0xF, q >> 4], axis=-1).reshape(q.shape[0], -1)
    vals = lib_e2m1_values()[codes]
    scales = lib_e4m3_values()[sf].repeat(16, axis=1)
    return vals, scales


@pytest.mark.parametrize("M,N,K,seed", [(4, 4, 32, 0), (8, 8, 64, 1), (3, 5, 48, 2)])
def test_gemm_exact_rationals(M, N, K, seed):
    rng = np.random.default_rng(seed)
    Aq, sfA = _random_operands(M, K, rng)
    Bq, sfB = _random_operands(N, K, rng)
    alpha = np.float32(0.7)
    v, S, exact = oracle.gemm(Aq, sfA, Bq, sfB, alpha)
    assert exact
    av, asf = _lib_deq(Aq, sfA)
    bv, bsf = _lib_deq(Bq, sfB)
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            s = Fraction(0)
            for k in range(K):
                p = (Fraction(av[m, k]) * Fraction(asf[m, k])) * (Fraction(bv[n, k]) * Fraction(bsf[n, k]))
                acc += p
                s += abs(p)
            assert v[m, n] == float(Fraction(float(alpha)) * acc)
            assert S[m, n] == float(s)


def test_gemm_zero_scales_give_zero():
    rng = np.random.default_rng(3)
    Aq, sfA = _random_operands(16, 256, rng)
    Bq, sfB = _random_operands(24, 256, rng)
    v, S, _ = oracle.gemm(Aq, np.zeros_like(sfA), Bq, sfB, 1.0)
    assert (v == 0).all() and (S == 0).all()


def test_gemm_one_hot_rows_reproduce_b_columns():
    rng = np.random.default_rng(4)
    M, N, K = 6, 40, 128
    Bq, sfB = _random_operands(N, K, rng)
    ks = [0, 1, 17, 64, 126, 127]
    Aq = np.zeros((M, K // 2), np.uint8)
    sfA = np.full((M, K // 16), 0x38, np.uint8)          # scale 1.0
    for m, k in enumerate(ks):
        Aq[m, k // 2] = 0x2 << (4 * (k % 2))              # code 2 = 1.0
    v, _, _ = oracle.gemm(Aq, sfA, Bq, sfB, 1.0)
    bv, bsf = _lib_deq(Bq, sfB)
    for m, k in enumerate(ks):
        np.testing.assert_array_equal(v[m], bv[:, k] * bsf[:, k])


def test_gemm_transpose_and_alpha_linearity():
    rng = np.random.default_rng(6)
    Aq, sfA = _random_operands(9, 256, rng)
    Bq, sfB = _random_operands(13, 256, rng)
    v1, S1, _ = oracle.gemm(Aq, sfA, Bq, sfB, 1.0)
    v2, S2, _ = oracle.gemm(Bq, sfB, Aq, sfA, 1.0)
    np.testing.assert_array_equal(v1, v2.T)
    np.testing.assert_array_equal(S1, S2.T)
    v3, _, _ = oracle.gemm(Aq, sfA, Bq, sfB, 2.0)
    np.testing.assert_array_equal(v3, 2.0 * v1)


def test_gemm_pipeline_approximates_fp64_product():
    rng = np.random.default_rng(8)
    a = rng.standard_normal((32, 512)).astype(np.float32)
    b = (rng.standard_normal((48, 512)) * 0.02).astype(np.float32)
    ga, gb = oracle.global_scale(a), oracle.global_scale(b)
    Aq, sfA = oracle.quantize(a, ga)
    Bq, sfB = oracle.quantize(b, gb)
    v, _, exact = oracle.gemm(Aq, sfA, Bq, sfB, oracle.alpha(ga, gb))
    ref = a.astype(np.float64) @ b.astype(np.float64).T
    assert exact
    rel = np.linalg.norm(v - ref) / np.linalg.norm(ref)
    assert rel < 0.15, rel            # 4-bit operands: ~10% normwise error is expected


def test_alpha_closed_form():
    assert oracle.alpha(448.0, 2.0) == np.float32(1.0 / 896.0)
    assert oracle.alpha(1.0, 1.0) == np.float32(1.0)


def test_grouped_gemm_matches_per_expert_products_and_rationals():
    rng = np.random.default_rng(12)
    E, N, K = 5, 16, 64
    counts = [3, 0, 5, 1, 0]
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(off[-1])
    Aq, sfA = _random_operands(rows, K, rng)
    Bq = rng.integers(0, 256, (E, N, K // 2), dtype=np.uint8)
    sfB = rng.integers(0x20, 0x48, (E, N, K // 16), dtype=np.uint8)
    alphas = rng.random(E).astype(np.float32)
    v, S, exact = oracle.grouped_gemm(Aq, sfA, Bq, sfB, alphas, off)
    assert exact
    for e in range(E):
        r0, r1 = off[e], off[e + 1]
        if r1 == r0:
            continue
        ve, Se, _ = oracle.gemm(Aq[r0:r1], sfA[r0:r1], Bq[e], sfB[e], alphas[e])
        np.testing.assert_array_equal(v[r0:r1], ve)
        np.testing.assert_array_equal(S[r0:r1], Se)
    # one element by exact rationals
    av, asf = _lib_deq(Aq, sfA)
    bv, bsf = _lib_deq(Bq[2], sfB[2])
    r, n = int(off[2]) + 4, 7
    acc = sum(Fraction(av[r, k]) * Fraction(asf[r, k]) * Fraction(bv[n, k]) * Fraction(bsf[n, k])
              for k in range(K))
    assert v[r, n] == float(Fraction(float(alphas[2])) * acc)


# ---------------------------------------------------------------- bf16 output rounding

def _bf16_brute(v):
    """Nearest bf16 to a double by exhaustive search of the bracketing pair."""
    f32 = np.float32(v)                        # only used to find a nearby bf16 pattern
    bits = int(np.array([f32], np.float32).view(np.uint32)[0]) >> 16
    cands = []
    for b in range(max(bits - 2, 0), min(bits + 3, 0xFFFF) + 1):
        if (b & 0x7F80) == 0x7F80:
            continue
        val = float(np.array([b << 16], np.uint32).view(np.float32)[0])
        cands.append((abs(val - v), b & 1, b))
    cands.sort()
    d0 = cands[0][0]
    tied = [c for c in cands if c[0] == d0]
    tied.sort(key=lambda c: c[1])             # prefer an even mantissa on ties
    return tied[0][2]


def test_bf16_rounding_brute_force():
    rng = np.random.default_rng(10)
    v = np.concatenate([rng.standard_normal(3000) * np.exp2(rng.integers(-20, 20, 3000)),
                        # values just off a bf16 midpoint, where rounding through fp32 first
                        # would differ from one direct rounding
                        np.array([1.0 + 2 ** -8 + 2 ** -30, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8,
                                  -(1.0 + 2 ** -8 + 2 ** -40)])])
    got = oracle.bf16_bits(v)
    for vi, gi in zip(v, got):
        want = _bf16_brute(float(abs(vi))) | (0x8000 if vi < 0 else 0)
        assert gi == want, (vi, hex(gi), hex(want))


def test_gemm_equals_gemm_of_dequantised_operands():
    # the benchmark's oracle leg dequantises the static weights once and calls
    # gemm_dequantized per step; gemm is defined as exactly that composition
    rng = np.random.default_rng(13)
    a = rng.standard_normal((9, 256)).astype(np.float32)
    b = rng.standard_normal((7, 256)).astype(np.float32)
    ga, gb = oracle.global_scale(a), oracle.global_scale(b)
    qa, sa = oracle.quantize(a, ga)
    qb, sb = oracle.quantize(b, gb)
    al = oracle.alpha(ga, gb)
    v, S, ex = oracle.gemm(qa, sa, qb, sb, al, threads=3)
    v2, S2, ex2 = oracle.gemm_dequantized(oracle.dequantize(qa, sa), oracle.dequantize(qb, sb), al, threads=2)
    np.testing.assert_array_equal(v, v2)
    np.testing.assert_array_equal(S, S2)
    assert ex and ex2


def test_fp16_rounding_matches_libraries_and_brute_force():
    """fp16 output option: one direct rounding of the fp64 value, against numpy's float64 ->
    float16 conversion and a nearest-value search over all finite fp16 values. (torch's
    conversion goes through fp32 first, two roundings, and differs near midpoints.)"""
    rng = np.random.default_rng(12)
    halves = np.arange(0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)   # +finite
    mids = (halves[:-1] + halves[1:]) / 2
    v = np.concatenate([rng.standard_normal(20000) * np.exp2(rng.integers(-26, 17, 20000)),
                        mids[::37], np.nextafter(mids[::41], 0), np.nextafter(mids[::43], np.inf),
                        [65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -24, 2.0 ** -25, 2.0 ** -26,
                         3 * 2.0 ** -26, 0.0, -0.0]])
    v = np.concatenate([v, -v])
    got = oracle.fp16_bits(v)
    with np.errstate(over="ignore"):          # 1e6 and 65520 overflow to inf, as intended
        np.testing.assert_array_equal(got, v.astype(np.float16).view(np.uint16))
    for vi in v[:400]:
        a = abs(float(vi))
        if a >= 65520.0:
            want = 0x7C00
        else:
            d = np.abs(halves - a)
            best = np.flatnonzero(d == d.min())
            want = int(best[0] if best.size == 1 else best[best % 2 == 0][0])
        want |= 0x8000 if np.signbit(vi) else 0
        assert oracle.fp16_bits(np.array([vi]))[0] == want, vi


# ---------------------------------------------------------------- frozen regression fixture

def test_oracle_regression_fixture():
    import json
    import os
    import sys
    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    sys.path.insert(0, here)
    import make_oracle_regression
    with open(os.path.join(here, "oracle_regression.json")) as f:
        stored = json.load(f)
    assert make_oracle_regression.compute() == stored


def test_oracle_next_regression_fixture():
    """The frozen results of the oracle's MXFP4, fp16, SwiGLU and routing functions; values
    that pass through exp are compared with a tolerance (libm implementations may differ in
    the last bit)."""
    import json
    import os
    import sys
    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    sys.path.insert(0, here)
    import make_oracle_next_regression
    with open(os.path.join(here, "oracle_next_regression.json")) as f:
        stored = json.load(f)
    got = make_oracle_next_regression.compute()
    for section in ("swiglu", "routing"):
        for key in ("h_samples", "weights_samples"):
            if key in stored[section]:
                np.testing.assert_allclose(got[section].pop(key), stored[section].pop(key), rtol=1e-14)
    assert got == stored
