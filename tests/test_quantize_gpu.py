"""GPU parity of the quantisation path (global scale, e4m3 block scales, e2m1 codes)
against the CPU oracle: bit-exact on every case, plus an exhaustive check of the two
rounding conversions over every finite fp32 bit pattern."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle
from helpers import gpu_quantize, oracle_quantize

pytestmark = pytest.mark.gpu


def _assert_same(xc, dev, dtype=torch.float32):
    q, sf, gs = gpu_quantize(xc, dev, dtype)
    qo, sfo, gso = oracle_quantize(xc, dtype)
    assert np.float32(gs.item()) == gso
    np.testing.assert_array_equal(sf.cpu().numpy(), sfo)
    np.testing.assert_array_equal(q.cpu().numpy(), qo)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_config_operands(cuda_device, dtype):
    cases = [workloads.single_case()] + workloads.attn_proj_cases() + workloads.moe_expert_cases()[:4]
    for c in cases:
        _assert_same(c.a(), cuda_device, dtype)
        _assert_same(c.b(), cuda_device, dtype)


def test_quantize_plateau_and_expert_weights(cuda_device):
    _assert_same(workloads.uniform(4096, 4096, 77), cuda_device)
    g = workloads.grouped_cases()[0]
    for e in (0, 255):
        _assert_same(g.b(e), cuda_device)
    _assert_same(g.a(64), cuda_device)


@pytest.mark.parametrize("rows,K", [(1, 16), (17, 48), (130, 256), (3, 6144), (257, 2048)])
def test_quantize_ragged_shapes(cuda_device, rows, K):
    _assert_same(workloads.normal(rows, K, 1.0, rows * 1000 + K), cuda_device)
    _assert_same(workloads.normal(rows, K, 1.0, rows * 1000 + K), cuda_device, torch.bfloat16)


def test_quantize_special_blocks(cuda_device):
    x = workloads.normal(8, 512, 1.0, 5)
    x[0] = 0.0                                   # zero row -> scales 0, codes 0
    x[1, :16] = 3.25                             # constant block
    x[2, 16:32] = torch.tensor([1e-30] * 16)     # tiny block (scale rounds to 0)
    x[3, 32:48] = -x[3, 32:48].abs()             # all-negative block
    x[4, 0] = 1e4                                # dominant element: others saturate towards 0
    x[5, :] = -0.0
    _assert_same(x, cuda_device)
    _assert_same(torch.zeros(4, 256), cuda_device)


def test_quantize_row_stride(cuda_device):
    xc = workloads.normal(40, 512, 1.0, 9)
    big = torch.zeros(40, 768)
    big[:, :512] = xc
    xd = big.to(cuda_device)[:, :512]
    gs = nv.global_scale(xd.contiguous())
    q, sf = nv.quantize(xd, gs)
    qo, sfo, _ = oracle_quantize(xc)
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(sf.cpu().numpy(), sfo)


def test_global_scale_edge_cases(cuda_device):
    z = torch.zeros(1000, device=cuda_device)
    assert nv.global_scale(z).item() == 1.0
    x = torch.tensor([1.0, -6.0, 2.0], device=cuda_device)
    assert nv.global_scale(x).item() == 448.0
    # numel not a multiple of the vector width: the tail must be reduced too
    xc = torch.zeros(1027)
    xc[1026] = -3.0
    assert nv.global_scale(xc.to(cuda_device)).item() == np.float32(2688.0) / np.float32(3.0)
    a = torch.tensor([3.0], device=cuda_device)
    b = torch.tensor([5.0, 7.0], device=cuda_device)
    al = nv.alpha(a, b).cpu().numpy()
    assert al[0] == oracle.alpha(3.0, 5.0) and al[1] == oracle.alpha(3.0, 7.0)


CHUNK = 1 << 28


def _finite_chunks():
    for start in range(0, 1 << 32, CHUNK):
        yield start


@pytest.mark.parametrize("kind", ["e4m3", "e2m1"])
def test_rounding_exhaustive_all_finite_fp32(cuda_device, kind):
    """Every finite fp32 bit pattern: GPU conversion == oracle conversion."""
    fn = nv.round_e4m3 if kind == "e4m3" else nv.round_e2m1
    enc = oracle.e4m3_encode if kind == "e4m3" else oracle.e2m1_encode
    for start in _finite_chunks():
        xh = np.arange(start, start + CHUNK, dtype=np.uint64).astype(np.uint32).view(np.float32)
        x = torch.from_numpy(xh).to(cuda_device)
        got = fn(x).cpu().numpy()
        finite = np.isfinite(xh)
        want = enc(xh)
        mism = (got != want) & finite
        if mism.any():
            i = np.argwhere(mism)[:5].ravel()
            raise AssertionError(f"{kind}: {int(mism.sum())} mismatches in chunk {start:#x}, e.g. "
                                 f"{[(float(xh[j]), int(got[j]), int(want[j])) for j in i]}")
        del x


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,K", [(1, 16), (16, 6144), (64, 6144), (1024, 6144), (17, 48),
                                    (257, 2048), (3, 16)])
def test_quantize_dynamic_matches_oracle(cuda_device, dtype, rows, K):
    xc = workloads.normal(rows, K, 1.0, rows * 31 + K)
    gb = torch.tensor([3.5, 700.25], device=cuda_device)
    q, sf, gs, al = nv.quantize_dynamic(xc.to(dtype).to(cuda_device), gs_other=gb)
    qo, sfo, gso = oracle_quantize(xc, dtype)
    assert np.float32(gs.item()) == gso
    np.testing.assert_array_equal(sf.cpu().numpy(), sfo)
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    al = al.cpu().numpy()
    assert al[0] == oracle.alpha(gso, 3.5) and al[1] == oracle.alpha(gso, 700.25)


def test_quantize_dynamic_zero_tensor_and_row_stride(cuda_device):
    q, sf, gs, al = nv.quantize_dynamic(torch.zeros(5, 256, device=cuda_device))
    assert gs.item() == 1.0 and al is None
    assert (q == 0).all() and (sf == 0).all()
    xc = workloads.normal(40, 512, 1.0, 19)
    big = torch.zeros(40, 640)
    big[:, :512] = xc
    q, sf, gs, _ = nv.quantize_dynamic(big.to(cuda_device)[:, :512])
    qo, sfo, gso = oracle_quantize(xc)
    assert np.float32(gs.item()) == gso
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(sf.cpu().numpy(), sfo)
