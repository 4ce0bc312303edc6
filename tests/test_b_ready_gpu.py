"""GPU checks of NVFP4_GEMM_B_READY (nvfp4_gemm_ex3): with the promise that no running kernel
writes B, the tiled-scale GEMM loads its first stages of B before waiting for the previous
kernel in the stream. The arithmetic is unchanged, so the output must equal the launch without
the flag bit for bit, on few-token (weights as the MMA M operand, split-K over a cluster),
mid-size and large shapes; each call follows the activation quantiser in the same stream, so
A is still being written when the GEMM's early loads start."""
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K", [(16, 768, 6144), (64, 6144, 2048), (40, 2048, 6144), (256, 768, 6144),
                                   (1024, 2048, 6144), (300, 776, 1024), (2048, 4096, 1024)])
def test_b_ready_same_bits(cuda_device, M, N, K):
    d = cuda_device
    a = workloads.normal(M, K, 1.0, 31 * M + N).to(d)
    b = workloads.normal(N, K, 0.02, 37 * N + K).to(d)
    gsB = nv.global_scale(b)
    Bq, sfB = nv.quantize(b, gsB)
    sfBt = nv.sf_tile(sfB)
    outs = []
    for ready in (False, True, True):
        q, sf, _, al = nv.quantize_dynamic(a, gs_other=gsB, tiled=True)
        outs.append(nv.gemm(q, sf, Bq, sfBt, al, workspace=nv.make_workspace(M, N, K, d), tiled=True,
                            b_ready=ready))
    st, code = nv.last_device_error()
    assert st == 0, hex(code)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    assert torch.equal(outs[0].view(torch.int16), outs[2].view(torch.int16))
