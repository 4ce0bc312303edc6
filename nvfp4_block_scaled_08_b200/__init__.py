"""nvfp4_block_scaled_08_b200 -- NVFP4 block-scaled matrix multiplication for B200 (sm_100a).

Thin Python binding over the C ABI of ``libnvfp4.so`` (``include/nvfp4.h``). Functions take
torch CUDA tensors for memory and the current CUDA stream, and only marshal pointers and
sizes: every step of quantisation and matrix multiplication runs in the library's CUDA
kernels. There is no CPU or alternative-backend path; if the library cannot be built or
loaded, or the device is not sm_100, calls raise.

    gs  = global_scale(x)                 # 2688 / max|x|  (fp32, device)
    q, sf = quantize(x, gs)               # packed e2m1 [R, K/2], e4m3 scales [R, K/16]
    al  = alpha(gs_a, gs_b)               # 1 / (gs_a * gs_b)
    gemm(Aq, sfA, Bq, sfB, al, out)       # out[M, N] bf16
    grouped_gemm(Aq, sfA, Bq, sfB, al_e, offsets, out)   # per-expert products

    # activations in one launch (global scale, alpha against the weights' scale, codes),
    # with the scales in the layout the tensor cores read; weights' scales re-laid out once
    q, sf, gs, al = quantize_dynamic(x, gs_other=gs_w, tiled=True)
    gemm(q, sf, Wq, sf_tile(sf_w), al, out, workspace=make_workspace(M, N, K), tiled=True)
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import _build

__all__ = [
    "Nvfp4Error", "load", "global_scale", "quantize", "quantize_dynamic", "alpha", "gemm", "gemm_workspace_size",
    "gemm_noalloc", "gemm_act", "plan_override",
    "make_workspace", "grouped_gemm", "grouped_gemm_swiglu", "moe_route", "moe_gather_quantize",
    "moe_combine", "mx_quantize", "mx_sf_tile", "mx_sf_bytes", "mx_gemm", "round_e4m3", "round_e2m1", "last_device_error",
    "STATUS",
]

STATUS = {
    0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_UNSUPPORTED_SHAPE",
    3: "NVFP4_ERR_MISALIGNED", 4: "NVFP4_ERR_ARCH", 5: "NVFP4_ERR_CUDA",
    6: "NVFP4_ERR_TIMEOUT", 7: "NVFP4_ERR_WORKSPACE",
}
IN_F32, IN_BF16 = 0, 1


class Nvfp4Error(RuntimeError):
    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn}: {message}")
        self.status = status


_lib = None
_lock = threading.Lock()

# exported symbol -> (restype, argtypes)
_P, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
SIGNATURES = {
    "nvfp4_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "nvfp4_global_scale": (ctypes.c_int, [_P, ctypes.c_int, _I64, _P, _P]),
    "nvfp4_quantize": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I64, _I64, _P, _P, _P, _P]),
    "nvfp4_alpha": (ctypes.c_int, [_P, _P, _I32, _P, _P]),
    "nvfp4_quantize_dynamic": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I64, _I64, _P, _P, _P, _P,
                                              _I32, _P, _P]),
    "nvfp4_gemm_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "nvfp4_gemm": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "nvfp4_gemm_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "nvfp4_check_bounded_wait": (ctypes.c_int, [ctypes.c_uint32, _P]),
    "nvfp4_quantize_dynamic_ex": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I64, _I64, _P, _P, _P, _P,
                                                 ctypes.c_int32, _P, ctypes.c_int, _P]),
    "nvfp4_sf_bytes": (_SZ, [_I64, _I64, ctypes.c_int]),
    "nvfp4_sf_tile": (ctypes.c_int, [_P, _I64, _I64, _P, _P]),
    "nvfp4_sf_8x4": (ctypes.c_int, [_P, _I64, _I64, _P, _P]),
    "nvfp4_gemm_ex": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, ctypes.c_int, _P]),
    "nvfp4_gemm_ex2": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, ctypes.c_int,
                                      ctypes.c_int, _P]),
    "nvfp4_gemm_ex3": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_uint32, _P]),
    "nvfp4_grouped_gemm_ex": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I32, _I64, _I64, _I64, _P,
                                             ctypes.c_int, _P]),
    "nvfp4_grouped_gemm_swiglu": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I32, _I64, _I64, _I64, _P, _P,
                                                 _P, _P]),
    "nvfp4_moe_route": (ctypes.c_int, [_P, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P]),
    "nvfp4_moe_gather_quantize": (ctypes.c_int, [_P, ctypes.c_int, _I32, _I64, _I64, _I32, _P, _P, _P, _P, _P,
                                                 _I32, _P, _P]),
    "nvfp4_moe_combine": (ctypes.c_int, [_P, ctypes.c_int, _P, _P, _I32, _I64, _I32, _P, ctypes.c_int, _P]),
    "nvfp4_mx_quantize": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I64, _I64, _P, _P, ctypes.c_int, _P]),
    "nvfp4_mx_sf_bytes": (_SZ, [_I64, _I64, ctypes.c_int]),
    "nvfp4_mx_sf_tile": (ctypes.c_int, [_P, _I64, _I64, _P, _P]),
    "nvfp4_mx_gemm": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, ctypes.c_int, _P]),
    "nvfp4_gemm_act": (ctypes.c_int, [_P, ctypes.c_int, _I64, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P,
                                      ctypes.c_int, _P]),
    "nvfp4_grouped_gemm_workspace_size": (_SZ, [_I32, _I64, _I64, _I64]),
    "nvfp4_grouped_gemm": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I32, _I64, _I64, _I64, _P, _P,
                                          _SZ, _P]),
    "nvfp4_set_plan_override": (ctypes.c_int, [_I32, _I32, _I32, _I32, _I32, _I32]),
    "nvfp4_round_e4m3": (ctypes.c_int, [_P, _I64, _P, _P]),
    "nvfp4_round_e2m1": (ctypes.c_int, [_P, _I64, _P, _P]),
    "nvfp4_last_device_error": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_uint32)]),
}


def library_path() -> str:
    return _build.LIB_PATH


def load(build_if_needed: bool = True) -> ctypes.CDLL:
    """Load libnvfp4.so (compiling it with nvcc first if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if build_if_needed:
            _build.build()
        if not os.path.exists(_build.LIB_PATH):
            raise Nvfp4Error("load", -1, f"CUDA library not found at {_build.LIB_PATH}")
        lib = ctypes.CDLL(_build.LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _check(fn: str, status: int):
    if status != 0:
        msg = load().nvfp4_status_string(status).decode()
        raise Nvfp4Error(fn, status, msg)


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def _dtype_code(x: torch.Tensor) -> int:
    if x.dtype == torch.float32:
        return IN_F32
    if x.dtype == torch.bfloat16:
        return IN_BF16
    raise ValueError("input must be float32 or bfloat16")


# ------------------------------------------------------------------ quantisation

def global_scale(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """gs = 2688 / max|x| (or 1 for an all-zero x) as a 1-element fp32 device tensor."""
    _dev(x, "x")
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    _check("nvfp4_global_scale", load().nvfp4_global_scale(
        _ptr(x), _dtype_code(x), x.numel(), _ptr(out), _stream(stream)))
    return out


def quantize(x: torch.Tensor, gs: torch.Tensor, q: torch.Tensor | None = None,
             sf: torch.Tensor | None = None, stream=None):
    """NVFP4 quantisation of x[rows, K] (fp32 or bf16, unit column stride).

    Returns (q uint8 [rows, K/2], sf uint8 [rows, K/16]) on x's device."""
    _dev(x, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    rows, K = x.shape
    if q is None:
        q = torch.empty(rows, K // 2, dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty(rows, K // 16, dtype=torch.uint8, device=x.device)
    _check("nvfp4_quantize", load().nvfp4_quantize(
        _ptr(x), _dtype_code(x), rows, K, x.stride(0), _ptr(gs), _ptr(q), _ptr(sf),
        _stream(stream)))
    return q, sf


SF_LINEAR, SF_TILED, SF_8X4 = 0, 1, 2


def _layout(tiled: bool, layout: int | None) -> int:
    """Scale layout code from the `tiled` flag or an explicit SF_* `layout` (which wins)."""
    if layout is None:
        return SF_TILED if tiled else SF_LINEAR
    if layout not in (SF_LINEAR, SF_TILED, SF_8X4):
        raise ValueError("layout must be SF_LINEAR, SF_TILED or SF_8X4")
    return layout


def sf_bytes(rows: int, K: int, tiled: bool = False, layout: int | None = None) -> int:
    return int(load().nvfp4_sf_bytes(rows, K, _layout(tiled, layout)))


def sf_tile(sf: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Row-major scales [rows, K/16] -> the tiled layout (flat uint8 tensor)."""
    rows, K = sf.shape[0], sf.shape[1] * 16
    if out is None:
        out = torch.empty(sf_bytes(rows, K, True), dtype=torch.uint8, device=sf.device)
    _check("nvfp4_sf_tile", load().nvfp4_sf_tile(_ptr(sf), rows, K, _ptr(out), _stream(stream)))
    return out


def sf_8x4(sf: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Row-major scales [rows, K/16] -> the 8 x 4 layout (flat uint8 tensor)."""
    rows, K = sf.shape[0], sf.shape[1] * 16
    if out is None:
        out = torch.empty(sf_bytes(rows, K, layout=SF_8X4), dtype=torch.uint8, device=sf.device)
    _check("nvfp4_sf_8x4", load().nvfp4_sf_8x4(_ptr(sf), rows, K, _ptr(out), _stream(stream)))
    return out


def quantize_dynamic(x: torch.Tensor, gs_other: torch.Tensor | None = None,
                     gs: torch.Tensor | None = None, q: torch.Tensor | None = None,
                     sf: torch.Tensor | None = None, alpha_out: torch.Tensor | None = None,
                     stream=None, tiled: bool = False, layout: int | None = None):
    """Global scale + quantisation (+ alpha against gs_other) in one launch; tiled: scales in
    the tiled layout (a flat uint8 tensor of sf_bytes(rows, K, True) bytes); layout: any SF_*
    layout (overrides tiled; SF_8X4 gives a flat tensor of sf_bytes(rows, K, layout=SF_8X4)).

    Returns (q, sf, gs, alpha) where alpha is None when gs_other is None."""
    _dev(x, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    rows, K = x.shape
    if q is None:
        q = torch.empty(rows, K // 2, dtype=torch.uint8, device=x.device)
    lay = _layout(tiled, layout)
    if sf is None:
        sf = (torch.empty(sf_bytes(rows, K, layout=lay), dtype=torch.uint8, device=x.device) if lay != SF_LINEAR
              else torch.empty(rows, K // 16, dtype=torch.uint8, device=x.device))
    if gs is None:
        gs = torch.empty(1, dtype=torch.float32, device=x.device)
    n = 0 if gs_other is None else gs_other.numel()
    if n and alpha_out is None:
        alpha_out = torch.empty(n, dtype=torch.float32, device=x.device)
    _check("nvfp4_quantize_dynamic_ex", load().nvfp4_quantize_dynamic_ex(
        _ptr(x), _dtype_code(x), rows, K, x.stride(0), _ptr(gs), _ptr(q), _ptr(sf),
        _ptr(gs_other), n, _ptr(alpha_out) if n else None, lay, _stream(stream)))
    return q, sf, gs, (alpha_out if n else None)


def alpha(gs_a: torch.Tensor, gs_b: torch.Tensor, out: torch.Tensor | None = None,
          stream=None) -> torch.Tensor:
    """alpha[i] = 1 / (gs_a[0] * gs_b[i]) (fp32, device)."""
    n = gs_b.numel()
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=gs_b.device)
    _check("nvfp4_alpha", load().nvfp4_alpha(_ptr(gs_a), _ptr(gs_b), n, _ptr(out),
                                             _stream(stream)))
    return out


# ------------------------------------------------------------------ products

def gemm_workspace_size(M: int, N: int, K: int) -> int:
    return int(load().nvfp4_gemm_workspace_size(M, N, K))


def make_workspace(M: int, N: int, K: int, device="cuda") -> torch.Tensor | None:
    """A zero-filled split-K workspace for this shape (None when none is needed)."""
    n = gemm_workspace_size(M, N, K)
    if n == 0:
        return None
    return torch.zeros(n, dtype=torch.uint8, device=device)


OUT_DTYPES = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2}


def _out_code(out: torch.Tensor) -> int:
    if out.dtype not in OUT_DTYPES:
        raise ValueError("out must be bfloat16, float16 or float32")
    return OUT_DTYPES[out.dtype]


def gemm(Aq, sfA, Bq, sfB, alpha_t, out=None, workspace=None, stream=None, tiled=False,
         out_dtype=torch.bfloat16, layout: int | None = None, b_ready: bool = False) -> torch.Tensor:
    """out[M, N] = alpha * sum_k deq(A)[m,k] deq(B)[n,k] in bf16, fp16 or fp32.

    Aq [M, K/2] uint8, sfA [M, K/16] uint8, Bq [N, K/2], sfB [N, K/16], alpha_t fp32 [1];
    out [M, N] (allocated with out_dtype if None; otherwise its dtype decides); workspace:
    zero-filled uint8 tensor of gemm_workspace_size(M, N, K) bytes or None (no split-K).
    tiled: sfA and sfB in the tiled layout (flat uint8 tensors from sf_tile or
    quantize_dynamic(tiled=True)); layout: any SF_* layout of both (overrides tiled).
    b_ready: NVFP4_GEMM_B_READY, a promise that no kernel that may still run writes Bq / sfB
    (weights quantised earlier): the kernel then loads its first stages of B before waiting
    for the previous kernel in the stream."""
    M, K = Aq.shape[0], Aq.shape[1] * 2
    N = Bq.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=Aq.device)
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (workspace.data_ptr(), workspace.numel())
    _check("nvfp4_gemm_ex3", load().nvfp4_gemm_ex3(
        _ptr(Aq), _ptr(sfA), _ptr(Bq), _ptr(sfB), _ptr(alpha_t), _ptr(out), M, N, K,
        ws_ptr, ws_bytes, _layout(tiled, layout), _out_code(out), 1 if b_ready else 0, _stream(stream)))
    return out


def gemm_act(x, gs_b, Bq, sfB_tiled, out=None, gs_out=None, alpha_out=None, stream=None,
             out_dtype=torch.bfloat16) -> torch.Tensor:
    """Few-token GEMM on unquantised activations x [M <= 64, K] (fp32 or bf16): the dynamic
    NVFP4 quantisation of x and the product in one launch (same bits as quantize_dynamic +
    gemm). Bq [N, K/2], sfB_tiled (tiled layout), gs_b fp32 [1] (the weights' global scale)."""
    _dev(x, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    M, K = x.shape
    N = Bq.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=x.device)
    _check("nvfp4_gemm_act", load().nvfp4_gemm_act(
        _ptr(x), _dtype_code(x), x.stride(0), _ptr(gs_b), _ptr(Bq), _ptr(sfB_tiled), _ptr(out), M, N, K,
        _ptr(gs_out), _ptr(alpha_out), _out_code(out), _stream(stream)))
    return out


def gemm_noalloc(Aq, sfA, Bq, sfB, alpha_t, out=None, stream=None) -> torch.Tensor:
    """Same product as gemm() for callers that cannot allocate device memory: the split-K
    scratch comes from a fixed array inside the library (no workspace argument). All calls
    on a device share that array, so calls must not overlap on the GPU. `out` must be given
    by such callers; allocating it here is a convenience for tests."""
    M, K = Aq.shape[0], Aq.shape[1] * 2
    N = Bq.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=Aq.device)
    _check("nvfp4_gemm_noalloc", load().nvfp4_gemm_noalloc(
        _ptr(Aq), _ptr(sfA), _ptr(Bq), _ptr(sfB), _ptr(alpha_t), _ptr(out), M, N, K,
        _stream(stream)))
    return out


def grouped_gemm(Aq, sfA, Bq, sfB, alphas, offsets, out=None, stream=None,
                 out_dtype=torch.bfloat16) -> torch.Tensor:
    """Per expert e: out[r] = alpha[e] * deq(A)[r] . deq(B[e])^T for rows r in
    [offsets[e], offsets[e+1]) (bf16, fp16 or fp32). Bq [E, N, K/2], sfB [E, N, K/16],
    offsets int32 [E+1]."""
    rows, K = Aq.shape[0], Aq.shape[1] * 2
    E, N = Bq.shape[0], Bq.shape[1]
    if out is None:
        out = torch.empty(rows, N, dtype=out_dtype, device=Aq.device)
    _check("nvfp4_grouped_gemm_ex", load().nvfp4_grouped_gemm_ex(
        _ptr(Aq), _ptr(sfA), _ptr(Bq), _ptr(sfB), _ptr(alphas), _ptr(offsets), E, rows, N, K,
        _ptr(out), _out_code(out), _stream(stream)))
    return out


class plan_override:
    """Context manager forcing parts of the GEMM launch plan (tuning and tests only):
    ``with plan_override(cluster=2, groups=3): ...``; the planner's choices return on exit."""

    def __init__(self, bn=0, cluster=0, groups=0, band=0, grouped_bn=0, pair=0):
        self.values = (bn, cluster, groups, band, grouped_bn, pair)

    def __enter__(self):
        _check("nvfp4_set_plan_override", load().nvfp4_set_plan_override(*self.values))
        return self

    def __exit__(self, *exc):
        _check("nvfp4_set_plan_override", load().nvfp4_set_plan_override(0, 0, 0, 0, 0, 0))
        return False


def grouped_gemm_swiglu(Aq, sfA, Bq, sfB, alphas, offsets, gs_h, h_q=None, h_sf=None, stream=None):
    """Grouped gate_up GEMM with SwiGLU and NVFP4 requantisation fused into the epilogue.

    Bq [E, 2I, K/2] (gate rows [0, I), up rows [I, 2I) per expert), sfB [E, 2I, K/16];
    gs_h fp32 [1] (device): the fixed global scale of h = silu(gate) * up.
    Returns (h_q uint8 [rows, I/2], h_sf uint8 [rows, I/16]), the down projection's A."""
    rows, K = Aq.shape[0], Aq.shape[1] * 2
    E, N = Bq.shape[0], Bq.shape[1]
    I = N // 2
    if h_q is None:
        h_q = torch.empty(rows, I // 2, dtype=torch.uint8, device=Aq.device)
    if h_sf is None:
        h_sf = torch.empty(rows, I // 16, dtype=torch.uint8, device=Aq.device)
    _check("nvfp4_grouped_gemm_swiglu", load().nvfp4_grouped_gemm_swiglu(
        _ptr(Aq), _ptr(sfA), _ptr(Bq), _ptr(sfB), _ptr(alphas), _ptr(offsets), E, rows, I, K,
        _ptr(gs_h), _ptr(h_q), _ptr(h_sf), _stream(stream)))
    return h_q, h_sf


# ------------------------------------------------------------------ MXFP4 (use_nvfp4=False)

def mx_sf_bytes(rows: int, K: int, tiled: bool = True) -> int:
    return int(load().nvfp4_mx_sf_bytes(rows, K, SF_TILED if tiled else SF_LINEAR))


def mx_quantize(x: torch.Tensor, q=None, sf=None, tiled: bool = True, stream=None):
    """MXFP4 quantisation of x[rows, K] (E8M0 scale per 32 elements, no per-tensor scale).
    Returns (q uint8 [rows, K/2], sf uint8: flat tiled scales, or [rows, K/32] if not tiled)."""
    _dev(x, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    rows, K = x.shape
    if q is None:
        q = torch.empty(rows, K // 2, dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = (torch.empty(mx_sf_bytes(rows, K, True), dtype=torch.uint8, device=x.device) if tiled
              else torch.empty(rows, K // 32, dtype=torch.uint8, device=x.device))
    _check("nvfp4_mx_quantize", load().nvfp4_mx_quantize(
        _ptr(x), _dtype_code(x), rows, K, x.stride(0), _ptr(q), _ptr(sf), SF_TILED if tiled else SF_LINEAR,
        _stream(stream)))
    return q, sf


def mx_sf_tile(sf: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Row-major MXFP4 scales [rows, K/32] -> the tiled layout (flat uint8 tensor)."""
    rows, K = sf.shape[0], sf.shape[1] * 32
    if out is None:
        out = torch.empty(mx_sf_bytes(rows, K, True), dtype=torch.uint8, device=sf.device)
    _check("nvfp4_mx_sf_tile", load().nvfp4_mx_sf_tile(_ptr(sf), rows, K, _ptr(out), _stream(stream)))
    return out


def mx_gemm(Aq, sfA, Bq, sfB, alpha_t, out=None, workspace=None, stream=None,
            out_dtype=torch.bfloat16) -> torch.Tensor:
    """MXFP4 product out[M, N] = alpha * sum_k deq(A) deq(B); sfA, sfB tiled E8M0 scales."""
    M, K = Aq.shape[0], Aq.shape[1] * 2
    N = Bq.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=Aq.device)
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (workspace.data_ptr(), workspace.numel())
    _check("nvfp4_mx_gemm", load().nvfp4_mx_gemm(
        _ptr(Aq), _ptr(sfA), _ptr(Bq), _ptr(sfB), _ptr(alpha_t), _ptr(out), M, N, K, ws_ptr, ws_bytes,
        _out_code(out), _stream(stream)))
    return out


# ------------------------------------------------------------------ mixture-of-experts layer

def moe_route(logits: torch.Tensor, k: int, experts=None, weights=None, offsets=None, row_of=None,
              token_of_row=None, stream=None):
    """Top-k routing of router logits [T, E] (fp32) and the expert-sorted permutation.

    Returns (experts int32 [T, k], weights fp32 [T, k], offsets int32 [E+1],
    row_of int32 [T, k], token_of_row int32 [T*k]) (allocated where not given)."""
    _dev(logits, "logits")
    if logits.dtype != torch.float32 or not logits.is_contiguous():
        raise ValueError("logits must be contiguous float32")
    T, E = logits.shape
    dev = logits.device
    if experts is None:
        experts = torch.empty(T, k, dtype=torch.int32, device=dev)
    if weights is None:
        weights = torch.empty(T, k, dtype=torch.float32, device=dev)
    if offsets is None:
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    if row_of is None:
        row_of = torch.empty(T, k, dtype=torch.int32, device=dev)
    if token_of_row is None:
        token_of_row = torch.empty(T * k, dtype=torch.int32, device=dev)
    _check("nvfp4_moe_route", load().nvfp4_moe_route(
        _ptr(logits), T, E, k, _ptr(experts), _ptr(weights), _ptr(offsets), _ptr(row_of),
        _ptr(token_of_row), _stream(stream)))
    return experts, weights, offsets, row_of, token_of_row


def moe_gather_quantize(x: torch.Tensor, row_of: torch.Tensor, gs_other: torch.Tensor | None = None,
                        gs=None, q=None, sf=None, alpha_out=None, stream=None):
    """Quantise tokens x [T, H] once (global scale over x) into their k expert-sorted rows.

    Returns (q uint8 [T*k, H/2], sf uint8 [T*k, H/16], gs, alpha or None)."""
    _dev(x, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    T, H = x.shape
    k = row_of.shape[1]
    dev = x.device
    if q is None:
        q = torch.empty(T * k, H // 2, dtype=torch.uint8, device=dev)
    if sf is None:
        sf = torch.empty(T * k, H // 16, dtype=torch.uint8, device=dev)
    if gs is None:
        gs = torch.empty(1, dtype=torch.float32, device=dev)
    n = 0 if gs_other is None else gs_other.numel()
    if n and alpha_out is None:
        alpha_out = torch.empty(n, dtype=torch.float32, device=dev)
    _check("nvfp4_moe_gather_quantize", load().nvfp4_moe_gather_quantize(
        _ptr(x), _dtype_code(x), T, H, x.stride(0), k, _ptr(row_of), _ptr(gs), _ptr(q), _ptr(sf),
        _ptr(gs_other), n, _ptr(alpha_out) if n else None, _stream(stream)))
    return q, sf, gs, (alpha_out if n else None)


def moe_combine(y: torch.Tensor, weights: torch.Tensor, row_of: torch.Tensor, out=None,
                out_dtype=torch.bfloat16, stream=None) -> torch.Tensor:
    """out[t] = sum_s weights[t, s] * y[row_of[t, s]] (fp32 accumulation, slot order)."""
    T, k = weights.shape
    H = y.shape[1]
    if out is None:
        out = torch.empty(T, H, dtype=out_dtype, device=y.device)
    if y.dtype not in OUT_DTYPES:
        raise ValueError("y must be bfloat16, float16 or float32")
    _check("nvfp4_moe_combine", load().nvfp4_moe_combine(
        _ptr(y), OUT_DTYPES[y.dtype], _ptr(weights), _ptr(row_of), T, H, k, _ptr(out), _out_code(out),
        _stream(stream)))
    return out


# ------------------------------------------------------------------ conversions and errors

def round_e4m3(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    _check("nvfp4_round_e4m3", load().nvfp4_round_e4m3(_ptr(x), x.numel(), _ptr(out),
                                                       _stream(stream)))
    return out


def round_e2m1(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    _check("nvfp4_round_e2m1", load().nvfp4_round_e2m1(_ptr(x), x.numel(), _ptr(out),
                                                       _stream(stream)))
    return out


def check_bounded_wait(timeout_us: int, stream=None) -> None:
    """Launch the bounded-wait check (a wait that must give up after timeout_us)."""
    _check("nvfp4_check_bounded_wait", load().nvfp4_check_bounded_wait(timeout_us, _stream(stream)))


def last_device_error(stream=None) -> tuple[int, int]:
    """(status, code) of the device error word, which is then cleared; synchronises."""
    where = ctypes.c_uint32(0)
    st = load().nvfp4_last_device_error(_stream(stream), ctypes.byref(where))
    return int(st), int(where.value)
