"""CPU checks of the C ABI: the library builds and loads without a GPU, exports every
function include/nvfp4.h declares, and rejects bad arguments on the host with the
documented status codes before any CUDA call is made."""
import ctypes
import os
import re

import pytest

import nvfp4_block_scaled_08_b200 as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "nvfp4.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return nv.load()


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for n in ("nvfp4_quantize", "nvfp4_gemm", "nvfp4_grouped_gemm", "nvfp4_global_scale",
              "nvfp4_last_device_error", "nvfp4_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(nv.SIGNATURES)


def test_status_strings(lib):
    for code, name in nv.STATUS.items():
        assert lib.nvfp4_status_string(code).decode().startswith(name)
    assert lib.nvfp4_status_string(99).decode() == "NVFP4_ERR_UNKNOWN"


def _gemm(lib, A=0x1000, sfA=0x2000, B=0x3000, sfB=0x4000, alpha=0x5000, out=0x6000,
          M=16, N=768, K=6144, ws=None, ws_bytes=0):
    return lib.nvfp4_gemm(A, sfA, B, sfB, alpha, out, M, N, K, ws, ws_bytes, None)


def test_gemm_host_validation(lib):
    # empty problems are a no-op and touch nothing
    assert _gemm(lib, M=0) == 0
    assert _gemm(lib, N=0) == 0
    assert _gemm(lib, M=-1) == 1
    assert _gemm(lib, A=None) == 1
    assert _gemm(lib, alpha=None) == 1
    assert _gemm(lib, out=None) == 1
    assert _gemm(lib, K=100) == 2          # K % 256
    assert _gemm(lib, K=0) == 2
    assert _gemm(lib, N=12) == 2           # N % 8
    assert _gemm(lib, M=1 << 31) == 2
    assert _gemm(lib, A=0x1001) == 3       # 16-byte alignment
    assert _gemm(lib, sfB=0x4008) == 3
    assert _gemm(lib, out=0x6002) == 3
    assert _gemm(lib, alpha=0x5002) == 3
    assert _gemm(lib, ws=0x7010, ws_bytes=1 << 20) == 3   # workspace needs 256-byte alignment


def _noalloc(lib, A=0x1000, sfA=0x2000, B=0x3000, sfB=0x4000, alpha=0x5000, out=0x6000,
             M=16, N=768, K=6144):
    return lib.nvfp4_gemm_noalloc(A, sfA, B, sfB, alpha, out, M, N, K, None)


@pytest.mark.parametrize("bad", [
    dict(M=0), dict(N=0), dict(M=-1), dict(K=-256), dict(A=None), dict(sfA=None), dict(B=None),
    dict(sfB=None), dict(alpha=None), dict(out=None), dict(K=100), dict(K=0), dict(N=12),
    dict(M=1 << 31), dict(N=1 << 31), dict(A=0x1001), dict(sfA=0x2004), dict(B=0x3008),
    dict(sfB=0x4008), dict(out=0x6002), dict(alpha=0x5002),
], ids=lambda d: ",".join(f"{k}={v}" for k, v in d.items()))
def test_noalloc_host_validation_matches_gemm(lib, bad):
    """The allocation-free entry point rejects every bad argument with the same status as
    nvfp4_gemm, before any CUDA call."""
    assert _noalloc(lib, **bad) == _gemm(lib, **bad)


def test_out_dtype_host_validation(lib):
    g = lib.nvfp4_gemm_ex2
    base = (0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 16, 768, 6144, None, 0, 0)
    assert g(*base, 3, None) == 1                    # bad out_dtype
    assert g(*base, -1, None) == 1
    assert g(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6008, 16, 768, 6144, None, 0, 0, 2, None) == 3
    gg = lib.nvfp4_grouped_gemm_ex
    args = (0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x8000, 256, 4096, 4096, 6144, 0x6000)
    assert gg(*args, 3, None) == 1
    assert gg(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x8000, 256, 4096, 4096, 6000, 0x6000, 1, None) == 2


def test_gemm_flags_host_validation(lib):
    g = lib.nvfp4_gemm_ex3
    base = (0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 16, 768, 6144, None, 0, 1, 0)
    assert g(*base, 2, None) == 1                    # unknown flag bit
    assert g(*base, 0x80000000, None) == 1
    assert g(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 16, 768, 6000, None, 0, 1, 0, 1, None) == 2


def test_mx_host_validation(lib):
    q = lib.nvfp4_mx_quantize
    assert q(0x1000, 0, 0, 512, 512, 0x2000, 0x3000, 0, None) == 0             # no rows
    assert q(0x1000, 0, 4, 48, 48, 0x2000, 0x3000, 0, None) == 2               # K % 32
    assert q(0x1000, 0, 4, 96, 96, 0x2000, 0x3000, 1, None) == 2               # tiled needs K % 128
    assert q(0x1000, 0, 4, 128, 128, 0x2000, 0x3000, 2, None) == 1             # bad layout
    assert q(0x1008, 0, 4, 128, 128, 0x2000, 0x3000, 0, None) == 3
    assert lib.nvfp4_mx_sf_bytes(300, 512, 0) == 300 * 16
    assert lib.nvfp4_mx_sf_bytes(300, 512, 1) == 384 * 16
    assert lib.nvfp4_mx_sf_bytes(300, 96, 1) == 0
    assert lib.nvfp4_mx_sf_tile(0x1000, 4, 96, 0x2000, None) == 2
    g = lib.nvfp4_mx_gemm
    assert g(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 16, 768, 6000, None, 0, 0, None) == 2
    assert g(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 16, 768, 6144, None, 0, 5, None) == 1
    assert g(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 0, 768, 6144, None, 0, 0, None) == 0


def test_moe_host_validation(lib):
    r = lib.nvfp4_moe_route
    assert r(0x1000, 4, 256, 8, 0x2000, 0x3000, None, 0x5000, 0x6000, None) == 1      # offsets
    assert r(0x1000, 4, 2048, 8, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None) == 2  # E > 1024
    assert r(0x1000, 4, 256, 33, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None) == 2  # k > 32
    assert r(0x1000, 4, 4, 8, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None) == 2     # k > E
    assert r(0x1002, 4, 256, 8, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None) == 3
    gq = lib.nvfp4_moe_gather_quantize
    assert gq(0x1000, 0, 0, 6144, 6144, 8, 0x2000, 0x3000, 0x4000, 0x5000, None, 0, None, None) == 2
    assert gq(0x1000, 0, 4, 6008, 6008, 8, 0x2000, 0x3000, 0x4000, 0x5000, None, 0, None, None) == 2
    assert gq(0x1008, 0, 4, 6144, 6144, 8, 0x2000, 0x3000, 0x4000, 0x5000, None, 0, None, None) == 3
    c = lib.nvfp4_moe_combine
    assert c(0x1000, 0, 0x2000, 0x3000, 4, 6144, 8, 0x4000, 3, None) == 1               # out dtype
    assert c(0x1000, 0, 0x2000, 0x3000, 4, 6148, 8, 0x4000, 0, None) == 2               # H % 8
    assert c(0x1000, 0, 0x2000, 0x3000, 0, 6144, 8, 0x4000, 0, None) == 0


def test_plan_override_validation(lib):
    assert lib.nvfp4_set_plan_override(-1, 0, 0, 0, 0, 0) == 1
    assert lib.nvfp4_set_plan_override(0, 0, -2, 0, 0, 0) == 1
    assert lib.nvfp4_set_plan_override(0, 0, 0, 0, 0, 4) == 1
    assert lib.nvfp4_set_plan_override(0, 0, 0, 0, 0, 0) == 0
    with nv.plan_override(cluster=2, groups=3):
        pass


def test_grouped_host_validation(lib):
    f = lib.nvfp4_grouped_gemm
    args = dict(A=0x1000, sfA=0x2000, B=0x3000, sfB=0x4000, alpha=0x5000, off=0x8000,
                E=256, rows=4096, N=4096, K=6144, out=0x6000)

    def call(**kw):
        a = dict(args, **kw)
        return f(a["A"], a["sfA"], a["B"], a["sfB"], a["alpha"], a["off"], a["E"], a["rows"],
                 a["N"], a["K"], a["out"], None, 0, None)

    assert call(E=0) == 0
    assert call(rows=0) == 0
    assert call(E=-1) == 1
    assert call(off=None) == 1
    assert call(E=2048) == 2               # more experts than the kernel supports
    assert call(K=6000) == 2
    assert call(off=0x8002) == 3
    assert call(B=0x3004) == 3
    assert lib.nvfp4_grouped_gemm_workspace_size(256, 4096, 4096, 6144) == 0


def test_quantize_host_validation(lib):
    q = lib.nvfp4_quantize
    assert q(0x1000, 0, 0, 6144, 6144, 0x2000, 0x3000, 0x4000, None) == 0   # no rows
    assert q(0x1000, 7, 4, 64, 64, 0x2000, 0x3000, 0x4000, None) == 1       # bad dtype
    assert q(None, 0, 4, 64, 64, 0x2000, 0x3000, 0x4000, None) == 1
    assert q(0x1000, 0, 4, 24, 24, 0x2000, 0x3000, 0x4000, None) == 2       # K % 16
    assert q(0x1000, 0, 4, 64, 32, 0x2000, 0x3000, 0x4000, None) == 1       # ld < K
    assert q(0x1008, 0, 4, 64, 64, 0x2000, 0x3000, 0x4000, None) == 3
    assert q(0x1000, 1, 4, 64, 68, 0x2000, 0x3000, 0x4000, None) == 3       # bf16 row stride 136 B
    gs = lib.nvfp4_global_scale
    assert gs(0x1000, 0, -1, 0x2000, None) == 1
    assert gs(0x1000, 0, 16, None, None) == 1
    assert gs(0x1004, 0, 16, 0x2000, None) == 3


def test_quantize_dynamic_host_validation(lib):
    f = lib.nvfp4_quantize_dynamic
    assert f(0x1000, 0, 4, 64, 64, None, 0x3000, 0x4000, None, 0, None, None) == 1     # gs_out
    assert f(0x1000, 0, 4, 64, 64, 0x2000, 0x3000, 0x4000, None, 2, 0x5000, None) == 1 # gs_other
    assert f(0x1000, 0, 0, 64, 64, 0x2000, 0x3000, 0x4000, None, 0, None, None) == 2   # empty
    assert f(0x1000, 0, 4, 24, 24, 0x2000, 0x3000, 0x4000, None, 0, None, None) == 2   # K % 16
    assert f(0x1004, 0, 4, 64, 64, 0x2000, 0x3000, 0x4000, None, 0, None, None) == 3


def test_tiled_scale_host_validation(lib):
    assert lib.nvfp4_sf_bytes(300, 512, 0) == 300 * 32
    assert lib.nvfp4_sf_bytes(300, 512, 1) == 384 * 32
    assert lib.nvfp4_sf_bytes(300, 48, 1) == 0          # tiled needs K % 64 == 0
    assert lib.nvfp4_sf_bytes(300, 512, 5) == 0
    assert lib.nvfp4_sf_tile(0x1000, 4, 48, 0x2000, None) == 2
    assert lib.nvfp4_sf_tile(None, 4, 64, 0x2000, None) == 1
    assert lib.nvfp4_sf_tile(0x1000, 0, 64, 0x2000, None) == 0
    g = lib.nvfp4_gemm_ex
    assert g(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 16, 768, 6144, None, 0, 7, None) == 1
    q = lib.nvfp4_quantize_dynamic_ex
    assert q(0x1000, 0, 4, 64, 64, 0x2000, 0x3000, 0x4000, None, 0, None, 3, None) == 1
    assert q(0x1000, 0, 4, 48, 48, 0x2000, 0x3000, 0x4000, None, 0, None, 1, None) == 2
    assert q(0x1000, 0, 4, 48, 48, 0x2000, 0x3000, 0x4000, None, 0, None, 2, None) == 2


def test_8x4_scale_host_validation(lib):
    assert lib.nvfp4_sf_bytes(300, 512, 2) == 304 * 32      # rows padded to 8
    assert lib.nvfp4_sf_bytes(8, 512, 2) == 8 * 32
    assert lib.nvfp4_sf_bytes(1, 64, 2) == 8 * 4
    assert lib.nvfp4_sf_bytes(300, 48, 2) == 0             # K % 64 == 0
    assert lib.nvfp4_sf_8x4(0x1000, 4, 48, 0x2000, None) == 2
    assert lib.nvfp4_sf_8x4(None, 4, 64, 0x2000, None) == 1
    assert lib.nvfp4_sf_8x4(0x1000, 4, 64, None, None) == 1
    assert lib.nvfp4_sf_8x4(0x1000, 0, 64, 0x2000, None) == 0
    assert lib.nvfp4_sf_8x4(0x1000, -1, 64, 0x2000, None) == 1
    g = lib.nvfp4_gemm_ex
    assert g(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 16, 768, 6000, None, 0, 2, None) == 2   # K % 256
    assert g(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 16, 768, 6144, None, 0, 3, None) == 1


def test_bounded_wait_check_host_validation(lib):
    assert lib.nvfp4_check_bounded_wait(0, None) == 1
    assert lib.nvfp4_check_bounded_wait(1000001, None) == 1


def test_round_and_alpha_host_validation(lib):
    assert lib.nvfp4_round_e4m3(None, 4, 0x1000, None) == 1
    assert lib.nvfp4_round_e2m1(0x1000, -1, 0x1000, None) == 1
    assert lib.nvfp4_round_e2m1(0x1000, 0, 0x1000, None) == 0
    assert lib.nvfp4_alpha(0x1000, 0x2000, 0, 0x3000, None) == 0
    assert lib.nvfp4_alpha(None, 0x2000, 1, 0x3000, None) == 1


def test_binding_is_argument_marshalling_only():
    # The binding must not import the oracle or compute anything itself.
    src = open(os.path.join(ROOT, "nvfp4_block_scaled_08_b200", "__init__.py")).read()
    assert "oracle" not in src.replace("no CPU or alternative-backend path", "")
    assert "import numpy" not in src


def test_build_tracks_every_source_and_header():
    """The library is rebuilt when any of its inputs is newer than it: every .cu file under
    csrc/ must be compiled and every header must be among the tracked inputs."""
    import os
    from nvfp4_block_scaled_08_b200 import _build
    files = set(os.listdir(_build.CSRC))
    assert {f for f in files if f.endswith(".cu")} == set(_build.SOURCES)
    assert {f for f in files if f.endswith((".cuh", ".h"))} == set(_build.HEADERS)
    tracked = {os.path.basename(p) for p in _build._inputs()}
    assert "nvfp4.h" in tracked and set(_build.SOURCES) | set(_build.HEADERS) <= tracked
