"""NVFP4_SF_TILED scales (include/nvfp4.h): the layout, the quantiser writing it, and the GEMM
reading it.

  * nvfp4_sf_tile against the layout formula, restated here in NumPy, byte for byte
    (padding rows zero);
  * nvfp4_quantize_dynamic_ex(..., TILED): the same codes, global scale and alpha as the
    linear call, and scales equal to the tiled image of the linear ones;
  * nvfp4_gemm_ex(..., TILED): bit-identical to nvfp4_gemm on the same scales in the linear
    layout (split-K, persistent multi-tile, ragged last tiles), and within the GEMM tolerance
    of the oracle on one shape.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle
from helpers import bf16_bits_of, check_within_tolerance, gpu_quantize, tile_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,K", [(1, 64), (128, 256), (300, 512), (1024, 6144)])
def test_sf_tile_matches_layout(cuda_device, rows, K):
    g = torch.Generator().manual_seed(rows + K)
    sf = torch.randint(0, 256, (rows, K // 16), dtype=torch.uint8, generator=g)
    t = nv.sf_tile(sf.to(cuda_device))
    assert t.numel() == nv.sf_bytes(rows, K, True) == (rows + 127) // 128 * 128 * K // 16
    assert np.array_equal(t.cpu().numpy(), tile_np(sf.numpy(), K))


@pytest.mark.parametrize("M,K,dtype", [(16, 6144, torch.float32), (64, 6144, torch.float32),
                                       (300, 512, torch.bfloat16), (1024, 6144, torch.float32)])
def test_quantize_dynamic_tiled_output(cuda_device, M, K, dtype):
    x = workloads.normal(M, K, 1.0, 7100 + M).to(dtype).to(cuda_device)
    gsb = torch.full((1,), 3.0, device=cuda_device)
    q0, sf0, gs0, al0 = nv.quantize_dynamic(x, gs_other=gsb)
    q1, sf1, gs1, al1 = nv.quantize_dynamic(x, gs_other=gsb, tiled=True)
    torch.cuda.synchronize()
    assert torch.equal(q0, q1) and torch.equal(gs0, gs1) and torch.equal(al0, al1)
    t = tile_np(sf0.cpu().numpy(), K)
    got = sf1.cpu().numpy()
    rows_pad = M % 128
    if rows_pad:   # padding bytes of the last row tile are not written by the quantiser
        mask = tile_np(np.ones((M, K // 16), np.uint8), K).astype(bool)
        assert np.array_equal(got[mask], t[mask])
    else:
        assert np.array_equal(got, t)


SHAPES = [(16, 768, 6144), (64, 768, 6144), (256, 768, 6144), (1024, 768, 6144),
          (512, 2048, 6144), (2048, 4096, 2048), (4096, 800, 512), (1, 256, 256), (200, 1000, 1024)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_tiled_equals_linear(cuda_device, M, N, K):
    d = cuda_device
    a = workloads.normal(M, K, 1.0, 7300 + M)
    b = workloads.normal(N, K, 0.02, 7400 + N)
    Aq, sfA, gsA = gpu_quantize(a, d)
    Bq, sfB, gsB = gpu_quantize(b, d)
    al = nv.alpha(gsA, gsB)
    ws = nv.make_workspace(M, N, K, d)
    ref = nv.gemm(Aq, sfA, Bq, sfB, al, workspace=ws)
    out = nv.gemm(Aq, nv.sf_tile(sfA), Bq, nv.sf_tile(sfB), al, workspace=ws, tiled=True)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits_of(out), bf16_bits_of(ref)), f"{M}x{N}x{K}"
    assert nv.last_device_error() == (0, 0)


def test_gemm_tiled_against_oracle(cuda_device):
    d = cuda_device
    case = workloads.attn_proj_cases()[2]
    a, b = case.a(), case.b()
    x = a.to(d)
    Bq, sfB, gsB = gpu_quantize(b, d)
    q, sf, gs, al = nv.quantize_dynamic(x, gs_other=gsB, tiled=True)
    out = nv.gemm(q, sf, Bq, nv.sf_tile(sfB), al, workspace=nv.make_workspace(case.M, case.N, case.K, d),
                  tiled=True)
    ga, gb = oracle.global_scale(a.numpy()), oracle.global_scale(b.numpy())
    qa, sa = oracle.quantize(a.numpy(), ga)
    qb, sb = oracle.quantize(b.numpy(), gb)
    alo = oracle.alpha(ga, gb)
    v, S, _ = oracle.gemm(qa, sa, qb, sb, alo)
    check_within_tolerance(out, v, S, alo, "tiled scales")
