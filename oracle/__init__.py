"""CPU oracle for NVFP4 block-scaled quantisation and matrix multiplication.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this module. The product path (``libnvfp4`` and the
``nvfp4_block_scaled_08_b200`` binding) never imports it and shares no code with it.

The arithmetic lives in ``nvfp4_oracle.c`` (plain C, fp64 accumulation, step-by-step
fp32 quantisation); this module builds it with gcc on first use and marshals numpy
arrays through ctypes. Every function states the passage of the reference pages it
follows; readings of points the pages leave open are listed in the design notes:

* e2m1 / e4m3 value tables and round-to-nearest-even encoders (the NVFP4 format:
  "When a Benchmark Crashes", section "Input Knowledge Required", item 3).
* ``global_scale`` / ``quantize``: the two-level NVFP4 recipe with 16-element blocks
  ("The Art of Reading the Manual", sections "The Message" and "Assumptions").
* ``gemm`` / ``grouped_gemm``: out = alpha * sum_k deq(A)[m,k] deq(B)[n,k], bf16 out
  ("The Moment the Zeros Disappeared", section "The Subject Message"); the grouped form
  is the per-expert product of a 256-expert, top-8 MoE layer ("When a Benchmark
  Crashes", section "Why This Message Was Written").
* ``route_topk`` / ``permute_by_expert`` / ``gather_quantize`` / ``combine``: the MoE
  layer's top-8-of-256 routing around the grouped product ("When a Benchmark Crashes",
  section "Why This Message Was Written"); readings at the functions. Not implemented by
  the CUDA library (the grouped product takes the sorted rows and offsets as inputs).
* ``silu`` / ``swiglu`` / ``swiglu_quantize``: the gate_up -> down step of the MoE expert
  MLP (intermediate 2048, "When a Benchmark Crashes", section "Why This Message Was
  Written"), SwiGLU then NVFP4 with a fixed global scale; readings at the function. Not
  implemented by the CUDA library.
* ``mx_quantize`` / ``mx_dequantize`` / ``mx_gemm``: the MXFP4 variant that the mm_fp4
  signature selects with ``use_nvfp4=False`` ("The Art of Reading the Manual", section "The
  Message"); the pages do not define it, so it follows the OCP MX v1.0 FP4 format (E8M0
  power-of-two scale per 32 elements, no per-tensor scale). Not implemented by the CUDA
  library.

Parity pins: ``tests/test_oracle.py``, ``tests/test_oracle_mx.py``,
``tests/test_oracle_swiglu.py`` and ``tests/test_oracle_routing.py`` (all functions pinned;
none is "parity unpinned").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-pthread"]


def build(force: bool = False) -> str:
    """Compile ``nvfp4_oracle.c`` into ``liboracle.so`` (gcc) if missing or stale."""
    with _lock:
        stale = (not os.path.exists(_LIB_PATH)
                 or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
        if force or stale:
            tmp = _LIB_PATH + ".%d.tmp" % os.getpid()
            subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
            os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    i64, i32, f32, f64, cint = (ctypes.c_int64, ctypes.c_int32, ctypes.c_float,
                                ctypes.c_double, ctypes.c_int)
    sig = {
        "oracle_e2m1_decode": (f64, [cint]),
        "oracle_e4m3_decode": (f64, [cint]),
        "oracle_e4m3_encode": (ctypes.c_uint8, [f32]),
        "oracle_e2m1_encode": (ctypes.c_uint8, [f32]),
        "oracle_e4m3_encode_array": (None, [P, i64, P, cint]),
        "oracle_e2m1_encode_array": (None, [P, i64, P, cint]),
        "oracle_global_scale": (f32, [P, i64]),
        "oracle_quantize": (None, [P, i64, i64, i64, f32, P, P]),
        "oracle_alpha": (f32, [f32, f32]),
        "oracle_dequantize": (None, [P, P, i64, i64, P]),
        "oracle_gemm_dequantized": (cint, [P, P, f64, i64, i64, i64, P, P, cint]),
        "oracle_gemm": (cint, [P, P, P, P, f32, i64, i64, i64, P, P, cint]),
        "oracle_grouped_gemm": (cint, [P, P, P, P, P, P, i32, i64, i64, P, P, cint]),
        "oracle_e8m0_decode": (f64, [cint]),
        "oracle_mx_quantize": (None, [P, i64, i64, i64, P, P]),
        "oracle_mx_dequantize": (None, [P, P, i64, i64, P]),
        "oracle_mx_gemm": (cint, [P, P, P, P, f32, i64, i64, i64, P, P, cint]),
        "oracle_bf16_bits": (ctypes.c_uint16, [f64]),
        "oracle_bf16_bits_array": (None, [P, i64, P]),
        "oracle_fp16_bits_array": (None, [P, i64, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _threads(n):
    return int(n) if n else (os.cpu_count() or 1)


# ---- format tables and encoders -------------------------------------------------------

def e2m1_decode(code: int) -> float:
    """Value of a 4-bit e2m1 code (sign, 2-bit exponent with bias 1, 1-bit mantissa)."""
    return _load().oracle_e2m1_decode(int(code))


def e4m3_decode(byte: int) -> float:
    """Value of an e4m3fn byte (bias 7, subnormals, 0x7F/0xFF NaN, max 448)."""
    return _load().oracle_e4m3_decode(int(byte))


def e4m3_encode(x, threads=None) -> np.ndarray:
    """fp32 -> e4m3fn bytes, round to nearest even, finite values saturate at +-448."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).reshape(-1)
    out = np.empty(x.size, dtype=np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(x), x.size, _ptr(out), _threads(threads))
    return out


def e2m1_encode(x, threads=None) -> np.ndarray:
    """fp32 -> e2m1 codes (0..15), nearest with ties to the even code, saturating at 6;
    the sign bit copies the input's sign (negative values rounding to 0 give 0x8)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).reshape(-1)
    out = np.empty(x.size, dtype=np.uint8)
    _load().oracle_e2m1_encode_array(_ptr(x), x.size, _ptr(out), _threads(threads))
    return out


# ---- quantisation ---------------------------------------------------------------------

def global_scale(x) -> np.float32:
    """gs = 2688 / max|x| (fp32), or 1 for an all-zero tensor (448 * 6 = 2688)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).reshape(-1)
    return np.float32(_load().oracle_global_scale(_ptr(x), x.size))


def quantize(x, gs) -> tuple[np.ndarray, np.ndarray]:
    """Two-level NVFP4 quantisation of a row-major fp32 [rows, K] tensor.

    Returns (q uint8 [rows, K/2], sf uint8 [rows, K/16]); element 2i sits in the low
    nibble of byte i; sf holds e4m3fn bytes.
    """
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    rows, K = x.shape
    assert K % 16 == 0
    q = np.empty((rows, K // 2), dtype=np.uint8)
    sf = np.empty((rows, K // 16), dtype=np.uint8)
    _load().oracle_quantize(_ptr(x), rows, K, K, float(np.float32(gs)), _ptr(q), _ptr(sf))
    return q, sf


def alpha(gs_a, gs_b) -> np.float32:
    """alpha = 1 / (gsA * gsB) in fp32."""
    return np.float32(_load().oracle_alpha(float(np.float32(gs_a)), float(np.float32(gs_b))))


def dequantize(q, sf) -> np.ndarray:
    """deq[r, k] = e2m1(q[r, k]) * e4m3(sf[r, k // 16]) as float64."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows, K = q.shape[0], q.shape[1] * 2
    out = np.empty((rows, K), dtype=np.float64)
    _load().oracle_dequantize(_ptr(q), _ptr(sf), rows, K, _ptr(out))
    return out


# ---- products -------------------------------------------------------------------------

def gemm(Aq, sfA, Bq, sfB, alpha_value, threads=None):
    """v = alpha * sum_k deq(A)[m,k] deq(B)[n,k] (fp64, ascending k, one rounding of
    the exact sum), S = sum_k |deq(A) deq(B)|. Returns (v, S, exact)."""
    Aq = np.ascontiguousarray(Aq, dtype=np.uint8)
    Bq = np.ascontiguousarray(Bq, dtype=np.uint8)
    sfA = np.ascontiguousarray(sfA, dtype=np.uint8)
    sfB = np.ascontiguousarray(sfB, dtype=np.uint8)
    M, K = Aq.shape[0], Aq.shape[1] * 2
    N = Bq.shape[0]
    assert Bq.shape[1] * 2 == K
    v = np.empty((M, N), dtype=np.float64)
    S = np.empty((M, N), dtype=np.float64)
    ex = _load().oracle_gemm(_ptr(Aq), _ptr(sfA), _ptr(Bq), _ptr(sfB),
                             float(np.float32(alpha_value)), M, N, K, _ptr(v), _ptr(S),
                             _threads(threads))
    if ex < 0:
        raise MemoryError("oracle_gemm: allocation failed")
    return v, S, bool(ex)


def gemm_dequantized(deqA, deqB, alpha_value, threads=None):
    """The sum of ``gemm`` on operands already dequantised (float64 [M, K] and [N, K]):
    ``gemm`` is dequantise-both then this. Returns (v, S, exact)."""
    deqA = np.ascontiguousarray(deqA, dtype=np.float64)
    deqB = np.ascontiguousarray(deqB, dtype=np.float64)
    M, K = deqA.shape
    N = deqB.shape[0]
    assert deqB.shape[1] == K
    v = np.empty((M, N), dtype=np.float64)
    S = np.empty((M, N), dtype=np.float64)
    ex = _load().oracle_gemm_dequantized(_ptr(deqA), _ptr(deqB), float(np.float32(alpha_value)), M, N, K,
                                         _ptr(v), _ptr(S), _threads(threads))
    return v, S, bool(ex)


def grouped_gemm(Aq, sfA, Bq, sfB, alphas, offsets, threads=None):
    """Per expert e: rows [off[e], off[e+1]) of A times B[e]^T, scaled by alpha[e].

    Bq is [E, N, K/2], sfB [E, N, K/16]; returns (v [rows, N], S, exact)."""
    Aq = np.ascontiguousarray(Aq, dtype=np.uint8)
    sfA = np.ascontiguousarray(sfA, dtype=np.uint8)
    Bq = np.ascontiguousarray(Bq, dtype=np.uint8)
    sfB = np.ascontiguousarray(sfB, dtype=np.uint8)
    alphas = np.ascontiguousarray(alphas, dtype=np.float32)
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    E, N, K = Bq.shape[0], Bq.shape[1], Bq.shape[2] * 2
    rows = Aq.shape[0]
    assert offsets.shape[0] == E + 1 and offsets[-1] <= rows
    v = np.zeros((rows, N), dtype=np.float64)
    S = np.zeros((rows, N), dtype=np.float64)
    ex = _load().oracle_grouped_gemm(_ptr(Aq), _ptr(sfA), _ptr(Bq), _ptr(sfB), _ptr(alphas),
                                     _ptr(offsets), E, N, K, _ptr(v), _ptr(S),
                                     _threads(threads))
    if ex < 0:
        raise MemoryError("oracle_grouped_gemm: allocation failed")
    return v, S, bool(ex)


# ---- MoE routing: top-k selection, expert-sorted permutation, combine ---------------------
# The layer routes every token to 8 of 256 experts ("When a Benchmark Crashes", section "Why
# This Message Was Written"); the pages do not give the router. Readings: probabilities are a
# softmax over the expert logits; a token takes the k largest, ties going to the lower expert
# index; its k weights are those probabilities renormalised to sum to 1; the expert-sorted
# order lists each expert's (token, slot) pairs in ascending token order; the combine after
# the down projection sums each token's k output rows weighted by its k weights.

def route_topk(logits, k: int):
    """logits fp32 [T, E] -> (experts int32 [T, k] by descending probability, probs fp64 [T, k],
    weights fp64 [T, k] = probs / probs.sum(row))."""
    z = np.asarray(logits, dtype=np.float64)
    z = z - z.max(axis=1, keepdims=True)
    p = np.exp(z)
    p = p / p.sum(axis=1, keepdims=True)
    order = np.argsort(-p, axis=1, kind="stable")[:, :k]     # stable: ties keep index order
    probs = np.take_along_axis(p, order, axis=1)
    return order.astype(np.int32), probs, probs / probs.sum(axis=1, keepdims=True)


def permute_by_expert(experts, num_experts: int):
    """experts int32 [T, k] -> (token_of_row int64 [T*k], slot_of_row int64 [T*k],
    offsets int32 [E + 1], row_of int64 [T, k]): rows of expert e are
    [offsets[e], offsets[e+1]), in ascending (token, slot) order; row_of[t, s] is the row
    that holds token t's slot s."""
    experts = np.asarray(experts)
    T, k = experts.shape
    flat = experts.reshape(-1).astype(np.int64)
    order = np.argsort(flat, kind="stable")                   # pair i = t * k + s
    counts = np.bincount(flat, minlength=num_experts)
    offsets = np.zeros(num_experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    row_of = np.empty(T * k, dtype=np.int64)
    row_of[order] = np.arange(T * k)
    return order // k, order % k, offsets, row_of.reshape(T, k)


def gather_quantize(x, token_of_row, gs):
    """The expert-sorted NVFP4 activations: the rows token_of_row of x, quantised with the
    tensor's global scale gs (rows are independent once gs is fixed)."""
    x = np.asarray(x, dtype=np.float32)
    return quantize(x[np.asarray(token_of_row)], gs)


def combine(y, weights, row_of):
    """out[t] = sum_s weights[t, s] * y[row_of[t, s]] in fp64, ascending s."""
    y = np.asarray(y, dtype=np.float64)
    weights = np.asarray(weights, dtype=np.float64)
    T, k = weights.shape
    out = np.zeros((T, y.shape[1]), dtype=np.float64)
    for s in range(k):
        out += weights[:, s:s + 1] * y[row_of[:, s]]
    return out


# ---- gate_up epilogue: SwiGLU, then NVFP4 requantisation for the down projection ----------
# The MoE layer's expert MLP ("When a Benchmark Crashes", section "Why This Message Was
# Written": intermediate size 2048) multiplies by a gate_up weight of 2 * 2048 rows and feeds
# down_proj. The pages do not spell out the activation between them; the readings here:
# columns [0, I) of the gate_up output are the gate g, columns [I, 2I) the up projection u,
# h = silu(g) * u with silu(g) = g / (1 + exp(-g)), evaluated in fp64 from the product's
# exact value, rounded once to fp32, and quantised to NVFP4 with a global scale fixed in
# advance (gs_h) rather than one taken from max|h|, which a GEMM epilogue cannot know.

def silu(g) -> np.ndarray:
    """silu(g) = g * sigmoid(g) = g / (1 + exp(-g)) in fp64 (exp(-g) overflows to inf for
    g < -709, giving -0.0 or 0.0, the limit)."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def swiglu(v) -> np.ndarray:
    """h = silu(g) * u for the gate_up output v [rows, 2I] (fp64): g = v[:, :I], u = v[:, I:]."""
    v = np.asarray(v, dtype=np.float64)
    I = v.shape[1] // 2
    assert v.shape[1] == 2 * I
    return silu(v[:, :I]) * v[:, I:]


def swiglu_quantize(v, gs_h) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """The gate_up epilogue: h = swiglu(v) rounded to fp32, then the NVFP4 steps of
    ``quantize`` with the fixed global scale gs_h. Returns (q, sf, h_fp32)."""
    h = swiglu(v).astype(np.float32)
    q, sf = quantize(h, gs_h)
    return q, sf, h


# ---- MXFP4 (use_nvfp4=False): OCP MX e2m1 with an E8M0 scale per 32 elements ------------

def e8m0_decode(byte: int) -> float:
    """Value of an E8M0 scale byte: 2^(byte - 127); 255 is NaN."""
    return _load().oracle_e8m0_decode(int(byte))


def mx_quantize(x) -> tuple[np.ndarray, np.ndarray]:
    """MXFP4 quantisation of a row-major fp32 [rows, K] tensor (K % 32 == 0): per 32-element
    block, shared_exp = floor(log2(amax)) - 2 clamped to [-127, 127] (all-zero block: -127),
    codes e2m1_rn_satfinite(x / 2^shared_exp). Returns (q uint8 [rows, K/2], sf uint8
    [rows, K/32] E8M0 bytes = shared_exp + 127)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    rows, K = x.shape
    assert K % 32 == 0
    q = np.empty((rows, K // 2), dtype=np.uint8)
    sf = np.empty((rows, K // 32), dtype=np.uint8)
    _load().oracle_mx_quantize(_ptr(x), rows, K, K, _ptr(q), _ptr(sf))
    return q, sf


def mx_dequantize(q, sf) -> np.ndarray:
    """deq[r, k] = e2m1(q[r, k]) * 2^(sf[r, k // 32] - 127) as float64."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows, K = q.shape[0], q.shape[1] * 2
    out = np.empty((rows, K), dtype=np.float64)
    _load().oracle_mx_dequantize(_ptr(q), _ptr(sf), rows, K, _ptr(out))
    return out


def mx_gemm(Aq, sfA, Bq, sfB, alpha_value=1.0, threads=None):
    """The MXFP4 product: v = alpha * sum_k deq(A)[m,k] deq(B)[n,k] with E8M0 scales per 32
    K elements (fp64, ascending k, one rounding of the exact sum), S = sum_k |a b|.
    Returns (v, S, exact)."""
    Aq = np.ascontiguousarray(Aq, dtype=np.uint8)
    Bq = np.ascontiguousarray(Bq, dtype=np.uint8)
    sfA = np.ascontiguousarray(sfA, dtype=np.uint8)
    sfB = np.ascontiguousarray(sfB, dtype=np.uint8)
    M, K = Aq.shape[0], Aq.shape[1] * 2
    N = Bq.shape[0]
    assert Bq.shape[1] * 2 == K and K % 32 == 0
    assert sfA.shape == (M, K // 32) and sfB.shape == (N, K // 32)
    v = np.empty((M, N), dtype=np.float64)
    S = np.empty((M, N), dtype=np.float64)
    ex = _load().oracle_mx_gemm(_ptr(Aq), _ptr(sfA), _ptr(Bq), _ptr(sfB),
                                float(np.float32(alpha_value)), M, N, K, _ptr(v), _ptr(S),
                                _threads(threads))
    if ex < 0:
        raise MemoryError("oracle_mx_gemm: allocation failed")
    return v, S, bool(ex)


def bf16_bits(v) -> np.ndarray:
    """Round float64 values to bf16 (nearest even, one rounding); raw uint16 bits."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    out = np.empty(v.shape, dtype=np.uint16)
    _load().oracle_bf16_bits_array(_ptr(v), v.size, _ptr(out))
    return out


def fp16_bits(v) -> np.ndarray:
    """Round float64 values to fp16 (nearest even, one rounding, inf above the range); raw
    uint16 bits. For the float16 output option of the product."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    out = np.empty(v.shape, dtype=np.uint16)
    _load().oracle_fp16_bits_array(_ptr(v), v.size, _ptr(out))
    return out


def tolerance(S, alpha_value) -> np.ndarray:
    """Allowed |out - v| per element: 2^-7 * |alpha| * sum_k |a b| + 1e-6."""
    return (2.0 ** -7) * abs(float(np.float32(alpha_value))) * np.asarray(S) + 1e-6
