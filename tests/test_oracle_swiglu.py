"""Pins for the oracle's gate_up epilogue (SwiGLU, then NVFP4 with a fixed global scale), the
step between the MoE expert's gate_up and down products ("When a Benchmark Crashes", section
"Why This Message Was Written": intermediate size 2048). Each check compares the oracle with
something other than itself:

* silu: scipy's logistic function (scipy.special.expit) times g, the identity
  silu(g) - silu(-g) = g, and its limits.
* swiglu: which half is the gate (h vanishes with the gate, not with the up projection; a
  large gate passes the up projection through).
* swiglu_quantize: an all-zero up projection gives zero codes and scales; the dequantised
  codes reconstruct h within the NVFP4 rounding bound of each 16-element block.
"""
import numpy as np
import pytest
import scipy.special

import oracle


def test_silu_matches_scipy_logistic():
    g = np.concatenate([np.linspace(-40, 40, 2001), np.array([-700.0, -1e-300, 0.0, 1e-300, 700.0]),
                        np.random.default_rng(0).standard_normal(5000) * 8])
    # a few ulps apart: two evaluation orders of the same function
    np.testing.assert_allclose(oracle.silu(g), g * scipy.special.expit(g), rtol=2e-15, atol=0)


def test_silu_identity_and_limits():
    g = np.random.default_rng(1).standard_normal(10000) * 10
    np.testing.assert_allclose(oracle.silu(g) - oracle.silu(-g), g, rtol=1e-15, atol=1e-300)
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(800.0) == 800.0
    assert oracle.silu(-800.0) == 0.0                      # exp overflow: the limit, -0.0
    assert oracle.silu(-20.0) == pytest.approx(-20.0 * np.exp(-20.0), rel=1e-8)


def test_swiglu_gate_is_the_first_half():
    I = 32
    rng = np.random.default_rng(2)
    u = rng.standard_normal((4, I))
    v = np.concatenate([np.zeros((4, I)), u], axis=1)           # gate 0: h = 0
    assert (oracle.swiglu(v) == 0).all()
    v = np.concatenate([np.full((4, I), 40.0), u], axis=1)      # gate 40: h = u (to 1e-16)
    np.testing.assert_allclose(oracle.swiglu(v), 40.0 * u, rtol=1e-15)
    v = np.concatenate([rng.standard_normal((4, I)), np.zeros((4, I))], axis=1)
    assert (oracle.swiglu(v) == 0).all()                        # up projection 0: h = 0


def test_swiglu_quantize_zero_up_projection():
    I = 64
    v = np.concatenate([np.random.default_rng(3).standard_normal((5, I)) * 3, np.zeros((5, I))], axis=1)
    q, sf, h = oracle.swiglu_quantize(v, np.float32(100.0))
    assert (h == 0).all() and (sf == 0).all() and ((q & 0x77) == 0).all()


@pytest.mark.parametrize("gs_h", [np.float32(2688.0 / 30.0), np.float32(64.0)])
def test_swiglu_quantize_reconstruction_bound(gs_h):
    I = 256
    rng = np.random.default_rng(4)
    v = rng.standard_normal((16, 2 * I)) * 4
    q, sf, h = oracle.swiglu_quantize(v, gs_h)
    np.testing.assert_array_equal(h, oracle.swiglu(v).astype(np.float32))
    deq = oracle.dequantize(q, sf) / np.float64(gs_h)
    scale = np.repeat(np.array([[oracle.e4m3_decode(b) for b in row] for row in sf]), 16, axis=1)
    step = scale / np.float64(gs_h)                 # one e2m1 unit (value 1.0) of the block
    y = np.abs(h.astype(np.float64)) / np.where(step > 0, step, np.inf)
    half = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0)) * step
    clip = np.maximum(y - 6.0, 0.0) * step
    # rounding of x * r to the e2m1 grid, plus the error of r = gs / scale itself (< 2^-23 rel)
    bound = np.maximum(half, clip) + np.abs(h) * 2.0 ** -20
    assert (np.abs(deq - h) <= bound).all()
