"""nvfp4_gemm_noalloc: the GEMM entry point for callers that cannot allocate device memory.

Who needs it: code running under a host framework that has reserved all device memory for
its own pool (a cudaMalloc there fails or fragments the framework's memory), interfaces
that hand a kernel no workspace argument, and latency-critical paths that cannot afford a
cudaMalloc / cudaFree that may synchronise the device. The entry point takes its split-K
scratch from a fixed array inside the library instead of a workspace.

Checked here, through the C ABI: two calls in a row give the same output as nvfp4_gemm
within the GEMM tolerance (2^-7 |alpha| sum|a b| + 1e-6 against the CPU oracle), both with
the default plan (which splits K inside one thread-block cluster and needs no scratch) and
with a plan forced to reduce split-K partials across several clusters, which goes through
the fixed scratch array and its tile counters; and a shape whose scratch would exceed the
fixed array is rejected with NVFP4_ERR_WORKSPACE. This file is collected last so that a
failure here cannot hide a failure elsewhere; it also passes when run on its own in a fresh
process.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle
from helpers import check_within_tolerance, gpu_quantize

pytestmark = pytest.mark.gpu

SENTINEL = -12352.0   # exactly representable in bf16


def _call_noalloc(lib, Aq, sfA, Bq, sfB, al, out, M, N, K):
    stream = torch.cuda.current_stream().cuda_stream
    return lib.nvfp4_gemm_noalloc(Aq.data_ptr(), sfA.data_ptr(), Bq.data_ptr(), sfB.data_ptr(),
                                  al.data_ptr(), out.data_ptr(), M, N, K, stream)


@pytest.mark.parametrize("case", workloads.attn_proj_cases()[:3] + workloads.moe_expert_cases()[1:2],
                         ids=lambda c: c.name)
@pytest.mark.parametrize("layout", ["planned", "workspace"])
def test_noalloc_matches_gemm_on_two_calls(cuda_device, case, layout):
    if layout == "workspace":
        # split-K across several clusters per tile, so the partials go through the scratch
        with nv.plan_override(cluster=2, groups=3):
            assert nv.gemm_workspace_size(case.M, case.N, case.K) > 0, "must use the scratch"
            _two_calls(cuda_device, case)
    else:
        # the default plan: no scratch (nothing for the fixed array to hold)
        assert nv.gemm_workspace_size(case.M, case.N, case.K) == 0
        _two_calls(cuda_device, case)


def _two_calls(cuda_device, case):
    d = cuda_device
    M, N, K = case.M, case.N, case.K
    a, b = case.a(), case.b()
    Aq, sfA, gsA = gpu_quantize(a, d)
    Bq, sfB, gsB = gpu_quantize(b, d)
    al = nv.alpha(gsA, gsB)
    ref = nv.gemm(Aq, sfA, Bq, sfB, al, workspace=nv.make_workspace(M, N, K, d))

    ga, gb = oracle.global_scale(a.numpy()), oracle.global_scale(b.numpy())
    qa, sa = oracle.quantize(a.numpy(), ga)
    qb, sb = oracle.quantize(b.numpy(), gb)
    alo = oracle.alpha(ga, gb)
    v, S, _ = oracle.gemm(qa, sa, qb, sb, alo)
    tol = oracle.tolerance(S, alo)
    ref_np = ref.float().cpu().numpy().astype(np.float64)

    lib = nv.load()
    for call in range(2):
        out = torch.full((M, N), SENTINEL, dtype=torch.bfloat16, device=d)
        st = _call_noalloc(lib, Aq, sfA, Bq, sfB, al, out, M, N, K)
        assert st == 0, lib.nvfp4_status_string(st).decode()
        st, code = nv.last_device_error()
        assert st == 0, hex(code)
        got = out.float().cpu().numpy().astype(np.float64)
        assert (np.abs(got - ref_np) <= tol).all(), f"call {call}: differs from nvfp4_gemm"
        check_within_tolerance(out, v, S, alo, f"{case.name} call {call}")


def test_noalloc_rejects_scratch_beyond_the_fixed_array(cuda_device):
    # force 24 cluster groups per tile on 1024 x 768 x 6144: 48 tiles x 24 x 64 KB > 16 MiB
    with nv.plan_override(cluster=1, groups=24):
        _rejects(cuda_device)


def _rejects(cuda_device):
    d = cuda_device
    M, N, K = 1024, 768, 6144
    Aq = torch.zeros(M, K // 2, dtype=torch.uint8, device=d)
    sfA = torch.zeros(M, K // 16, dtype=torch.uint8, device=d)
    Bq = torch.zeros(N, K // 2, dtype=torch.uint8, device=d)
    sfB = torch.zeros(N, K // 16, dtype=torch.uint8, device=d)
    al = torch.ones(1, device=d)
    out = torch.full((M, N), SENTINEL, dtype=torch.bfloat16, device=d)
    lib = nv.load()
    st = _call_noalloc(lib, Aq, sfA, Bq, sfB, al, out, M, N, K)
    assert st == 7, lib.nvfp4_status_string(st).decode()          # NVFP4_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (out.float() == SENTINEL).all(), "a rejected call must not launch anything"
