"""GPU checks of nvfp4_gemm_act: the few-token GEMM that quantises its fp32 / bf16 activations
inside the kernel (every CTA of the split-K cluster quantises its own K slice, the slices'
maxima meet over distributed shared memory).

The codes, scales, alpha and MMAs are those of nvfp4_quantize_dynamic_ex followed by
nvfp4_gemm_ex2, so the output must equal that two-launch path bit for bit, and gs / alpha must
equal the oracle's; the product is also held to the GEMM tolerance of the CPU oracle
(2^-7 |alpha| sum|a b| + 1e-6). Shapes: the decode configurations (M = 16 ... 64), ragged
token counts (1, 17, 33), an all-zero activation tensor (global scale 1), bf16 input, a row
stride larger than K, fp32 output, and a shape whose K slices do not fit the stage ring
(rejected)."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle
from helpers import check_within_tolerance

pytestmark = pytest.mark.gpu


def _weights(dev, b):
    bd = b.to(dev)
    gs = nv.global_scale(bd)
    q, sf = nv.quantize(bd, gs)
    return q, nv.sf_tile(sf), gs


def _two_launch(x, Bq, sfBt, gsB, out_dtype):
    q, sf, gs, al = nv.quantize_dynamic(x, gs_other=gsB, tiled=True)
    M, K = x.shape
    out = nv.gemm(q, sf, Bq, sfBt, al, workspace=nv.make_workspace(M, Bq.shape[0], K, x.device), tiled=True,
                  out_dtype=out_dtype)
    return out, gs, al


def _check(dev, a, b, dtype=torch.float32, out_dtype=torch.bfloat16, ld_pad=0):
    M, K = a.shape
    N = b.shape[0]
    Bq, sfBt, gsB = _weights(dev, b)
    xa = a.to(dtype)
    if ld_pad:
        big = torch.zeros(M, K + ld_pad, dtype=dtype)
        big[:, :K] = xa
        x = big.to(dev)[:, :K]
    else:
        x = xa.to(dev)
    gs_out = torch.full((1,), -1.0, device=dev)
    al_out = torch.full((1,), -1.0, device=dev)
    out = nv.gemm_act(x, gsB, Bq, sfBt, gs_out=gs_out, alpha_out=al_out, out_dtype=out_dtype)
    st, code = nv.last_device_error()
    assert st == 0, hex(code)
    ref, gs2, al2 = _two_launch(x, Bq, sfBt, gsB, out_dtype)
    assert torch.equal(out.view(torch.int16 if out.element_size() == 2 else torch.int32),
                       ref.view(torch.int16 if ref.element_size() == 2 else torch.int32)), "differs from the two launches"
    x32 = xa.to(torch.float32).numpy()
    ga, gb = oracle.global_scale(x32), oracle.global_scale(b.numpy())
    assert np.float32(gs_out.item()) == ga and torch.equal(gs_out, gs2)
    alo = oracle.alpha(ga, gb)
    assert np.float32(al_out.item()) == alo and torch.equal(al_out, al2)
    qa, sa = oracle.quantize(x32, ga)
    qb, sb = oracle.quantize(b.numpy(), gb)
    v, S, _ = oracle.gemm(qa, sa, qb, sb, alo)
    check_within_tolerance(out, v, S, alo, f"gemm_act {M}x{N}x{K}")


@pytest.mark.parametrize("case", [c for c in workloads.attn_proj_cases() + workloads.moe_expert_cases() if c.M <= 64],
                         ids=lambda c: c.name)
def test_decode_configs(cuda_device, case):
    _check(cuda_device, case.a(), case.b())


@pytest.mark.parametrize("M,N,K", [(1, 768, 6144), (17, 264, 2048), (33, 1024, 4096), (64, 136, 1024)])
def test_ragged(cuda_device, M, N, K):
    _check(cuda_device, workloads.normal(M, K, 1.0, M + N), workloads.normal(N, K, 0.02, N + K))


def test_bf16_input_row_stride_and_fp32_out(cuda_device):
    a = workloads.normal(24, 2048, 1.0, 5)
    b = workloads.normal(512, 2048, 0.02, 6)
    _check(cuda_device, a, b, dtype=torch.bfloat16, ld_pad=64)
    _check(cuda_device, a, b, out_dtype=torch.float32)


def test_all_zero_activations(cuda_device):
    a = torch.zeros(16, 6144)
    b = workloads.normal(768, 6144, 0.02, 7)
    _check(cuda_device, a, b)


def test_rejects_slices_beyond_the_ring(cuda_device):
    # 64 tokens, N = 32768: 256 weight tiles leave no room for split-K, one CTA would hold all
    # 24 K stages of K = 6144
    d = cuda_device
    x = torch.zeros(64, 6144, device=d)
    Bq = torch.zeros(32768, 3072, dtype=torch.uint8, device=d)
    sfB = torch.zeros(nv.sf_bytes(32768, 6144, True), dtype=torch.uint8, device=d)
    with pytest.raises(nv.Nvfp4Error) as e:
        nv.gemm_act(x, torch.ones(1, device=d), Bq, sfB)
    assert e.value.status == 2
