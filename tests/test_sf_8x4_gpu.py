"""NVFP4_SF_8X4 scales (include/nvfp4.h): the layout, the quantiser writing it, and the dense
GEMM reading it.

  * nvfp4_sf_8x4 against the layout formula, restated here in NumPy, byte for byte (padding
    rows zero);
  * nvfp4_quantize_dynamic_ex(..., 8X4): the same codes, global scale and alpha as the linear
    call, and scales equal to the 8 x 4 image of the linear ones (real rows; the quantiser
    leaves padding bytes alone);
  * nvfp4_gemm_ex(..., 8X4): bit-identical to nvfp4_gemm on the same scales in the linear
    layout (few-token tiles with and without split-K, 128/192/224/256-wide tiles, persistent
    multi-tile, ragged last tiles, fp32 output), and within the GEMM tolerance of the oracle
    on a decode shape quantised straight into the 8 x 4 layout.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle
from helpers import bf16_bits_of, check_within_tolerance, gpu_quantize, layout_8x4_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,K", [(1, 64), (7, 256), (8, 256), (37, 512), (300, 512), (1024, 6144)])
def test_sf_8x4_matches_layout(cuda_device, rows, K):
    g = torch.Generator().manual_seed(rows + 3 * K)
    sf = torch.randint(0, 256, (rows, K // 16), dtype=torch.uint8, generator=g)
    t = nv.sf_8x4(sf.to(cuda_device))
    assert t.numel() == nv.sf_bytes(rows, K, layout=nv.SF_8X4) == (rows + 7) // 8 * 8 * K // 16
    assert np.array_equal(t.cpu().numpy(), layout_8x4_np(sf.numpy(), K))


@pytest.mark.parametrize("M,K,dtype", [(1, 6144, torch.float32), (13, 6144, torch.bfloat16),
                                       (64, 2048, torch.float32), (300, 512, torch.bfloat16),
                                       (4096, 6144, torch.float32)])
def test_quantize_dynamic_8x4_output(cuda_device, M, K, dtype):
    x = workloads.normal(M, K, 1.0, 7700 + M).to(dtype).to(cuda_device)
    gsb = torch.full((1,), 3.0, device=cuda_device)
    q0, sf0, gs0, al0 = nv.quantize_dynamic(x, gs_other=gsb)
    q1, sf1, gs1, al1 = nv.quantize_dynamic(x, gs_other=gsb, layout=nv.SF_8X4)
    torch.cuda.synchronize()
    assert torch.equal(q0, q1) and torch.equal(gs0, gs1) and torch.equal(al0, al1)
    assert sf1.numel() == nv.sf_bytes(M, K, layout=nv.SF_8X4)
    want = layout_8x4_np(sf0.cpu().numpy(), K)
    mask = layout_8x4_np(np.ones((M, K // 16), np.uint8), K).astype(bool)
    assert np.array_equal(sf1.cpu().numpy()[mask], want[mask])


SHAPES = [(1, 256, 256), (5, 768, 6144), (16, 768, 6144), (37, 1024, 2048), (64, 6144, 2048),
          (128, 768, 6144), (200, 1000, 1024), (512, 2048, 6144), (2048, 4096, 2048), (4096, 800, 512)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_8x4_equals_linear(cuda_device, M, N, K):
    d = cuda_device
    a = workloads.normal(M, K, 1.0, 7800 + M)
    b = workloads.normal(N, K, 0.02, 7900 + N)
    Aq, sfA, gsA = gpu_quantize(a, d)
    Bq, sfB, gsB = gpu_quantize(b, d)
    al = nv.alpha(gsA, gsB)
    sA, sB = nv.sf_8x4(sfA), nv.sf_8x4(sfB)
    for ws in (nv.make_workspace(M, N, K, d), None):
        ref = nv.gemm(Aq, sfA, Bq, sfB, al, workspace=ws)
        out = nv.gemm(Aq, sA, Bq, sB, al, workspace=ws, layout=nv.SF_8X4)
        torch.cuda.synchronize()
        assert np.array_equal(bf16_bits_of(out), bf16_bits_of(ref)), f"{M}x{N}x{K} ws={ws is not None}"
    ref32 = nv.gemm(Aq, sfA, Bq, sfB, al, out_dtype=torch.float32)
    out32 = nv.gemm(Aq, sA, Bq, sB, al, out_dtype=torch.float32, layout=nv.SF_8X4)
    assert torch.equal(out32.view(torch.int32), ref32.view(torch.int32))
    assert nv.last_device_error() == (0, 0)


@pytest.mark.parametrize("bn", [128, 192, 224, 256])
def test_gemm_8x4_every_tile_width(cuda_device, bn):
    d = cuda_device
    M, N, K = 300, 1000, 1024
    a = workloads.normal(M, K, 1.0, 8100 + bn)
    b = workloads.normal(N, K, 0.02, 8200 + bn)
    Aq, sfA, gsA = gpu_quantize(a, d)
    Bq, sfB, gsB = gpu_quantize(b, d)
    al = nv.alpha(gsA, gsB)
    with nv.plan_override(bn=bn):
        ref = nv.gemm(Aq, sfA, Bq, sfB, al)
        out = nv.gemm(Aq, nv.sf_8x4(sfA), Bq, nv.sf_8x4(sfB), al, layout=nv.SF_8X4)
        torch.cuda.synchronize()
    assert np.array_equal(bf16_bits_of(out), bf16_bits_of(ref)), f"bn={bn}"
    assert nv.last_device_error() == (0, 0)


def test_gemm_8x4_against_oracle(cuda_device):
    d = cuda_device
    case = workloads.attn_proj_cases()[1]
    a, b = case.a(), case.b()
    Bq, sfB, gsB = gpu_quantize(b, d)
    q, sf, gs, al = nv.quantize_dynamic(a.to(d), gs_other=gsB, layout=nv.SF_8X4)
    out = nv.gemm(q, sf, Bq, nv.sf_8x4(sfB), al, workspace=nv.make_workspace(case.M, case.N, case.K, d),
                  layout=nv.SF_8X4)
    ga, gb = oracle.global_scale(a.numpy()), oracle.global_scale(b.numpy())
    qa, sa = oracle.quantize(a.numpy(), ga)
    qb, sb = oracle.quantize(b.numpy(), gb)
    alo = oracle.alpha(ga, gb)
    v, S, _ = oracle.gemm(qa, sa, qb, sb, alo)
    check_within_tolerance(out, v, S, alo, "8x4 scales")
