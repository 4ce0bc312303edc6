"""GPU parity of the mixture-of-experts layer around the grouped GEMM against the CPU oracle
(oracle.route_topk, oracle.permute_by_expert, oracle.gather_quantize, oracle.combine): the
top-8-of-256 routing of "When a Benchmark Crashes", section "Why This Message Was Written".

* Routing: the expert indices, the expert offsets, the row of every (token, slot) pair and the
  token of every sorted row are integer results and must be bit-exact, ties included (ties go
  to the lower expert index). The weights are computed in fp32 with CUDA's expf: within
  2^-20 of the oracle's fp64 values (they lie in (0, 1]; a handful of fp32 roundings and
  expf's few ulp stay far below that).
* Gather-quantise: the codes, scales, global scale and alphas are bit-exact (the same fp32
  operations as the quantiser, whose exactness the quantiser tests pin), in both launch forms
  (one thread-block cluster for small inputs, a cooperative grid for large ones).
* Combine: both sides get the same fp32 weights and the same y; the kernel sums k fp32
  products in slot order, so |out - v| <= (k + 2) 2^-24 sum_s |w_s y_s| for fp32 output, plus
  the output type's rounding, at most its unit roundoff times |v| (2^-8 for bf16's 8
  significant bits, 2^-11 for fp16's 11).
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle

pytestmark = pytest.mark.gpu


def _route_both(dev, logits: torch.Tensor, k: int):
    E = logits.shape[1]
    ex, w, off, row_of, tok = nv.moe_route(logits.to(dev), k)
    st, code = nv.last_device_error()
    assert st == 0, hex(code)
    ex_o, probs_o, w_o = oracle.route_topk(logits.numpy(), k)
    tok_o, slot_o, off_o, row_o = oracle.permute_by_expert(ex_o, E)
    return (ex.cpu().numpy(), w.cpu().numpy(), off.cpu().numpy(), row_of.cpu().numpy(), tok.cpu().numpy(),
            ex_o, w_o, off_o, row_o, tok_o)


@pytest.mark.parametrize("T,E,k", [(1, 256, 8), (37, 256, 8), (512, 256, 8), (4096, 256, 8), (300, 100, 6),
                                   (64, 64, 32), (129, 1024, 8), (50, 33, 1)])
def test_route_matches_oracle(cuda_device, T, E, k):
    logits = workloads.normal(T, E, 1.0, 1000 + T + E + k)
    ex, w, off, row_of, tok, ex_o, w_o, off_o, row_o, tok_o = _route_both(cuda_device, logits, k)
    np.testing.assert_array_equal(ex, ex_o)
    np.testing.assert_array_equal(off, off_o)
    np.testing.assert_array_equal(row_of, row_o)
    np.testing.assert_array_equal(tok, tok_o)
    assert np.abs(w - w_o).max() <= 2.0 ** -20
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-6)


def test_route_ties_go_to_the_lower_expert(cuda_device):
    # logits on a coarse grid: many exact ties inside every token's top 8
    logits = torch.round(workloads.normal(200, 256, 1.0, 77) * 2.0) / 2.0
    ex, w, off, row_of, tok, ex_o, w_o, off_o, row_o, tok_o = _route_both(cuda_device, logits, 8)
    np.testing.assert_array_equal(ex, ex_o)
    np.testing.assert_array_equal(row_of, row_o)
    np.testing.assert_array_equal(off, off_o)
    assert np.abs(w - w_o).max() <= 2.0 ** -20
    # all-equal logits: every token takes experts 0..7 with weights 1/8
    flat = torch.zeros(16, 256)
    ex, w, off, *_ = _route_both(cuda_device, flat, 8)
    assert (ex == np.arange(8)).all() and np.allclose(w, 0.125)
    assert off[8] == 16 * 8 and off[-1] == 16 * 8


def test_route_no_tokens(cuda_device):
    lib = nv.load()
    off = torch.full((257,), 7, dtype=torch.int32, device=cuda_device)
    dummy = torch.zeros(8, dtype=torch.int32, device=cuda_device)
    st = lib.nvfp4_moe_route(dummy.data_ptr(), 0, 256, 8, dummy.data_ptr(), dummy.data_ptr(), off.data_ptr(),
                             dummy.data_ptr(), dummy.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    assert (off == 0).all()


@pytest.mark.parametrize("T,H,dtype", [(16, 512, torch.float32), (64, 6144, torch.bfloat16),
                                       (512, 6144, torch.float32), (4096, 6144, torch.float32),
                                       (100, 2048, torch.bfloat16)])
def test_gather_quantize_bit_exact(cuda_device, T, H, dtype):
    d = cuda_device
    E, k = 256, 8
    logits = workloads.normal(T, E, 1.0, 5000 + T)
    ex_o, _, _ = oracle.route_topk(logits.numpy(), k)
    tok_o, _, off_o, row_o = oracle.permute_by_expert(ex_o, E)
    x = workloads.normal(T, H, 1.0, 6000 + T + H).to(dtype)
    gs_w = (torch.rand(E, generator=torch.Generator().manual_seed(3)) * 100 + 1).float()
    q, sf, gs, al = nv.moe_gather_quantize(x.to(d), torch.from_numpy(row_o.astype(np.int32)).to(d),
                                           gs_other=gs_w.to(d))
    st, code = nv.last_device_error()
    assert st == 0, hex(code)
    x32 = x.to(torch.float32).numpy()
    ga = oracle.global_scale(x32)
    q_o, sf_o = oracle.gather_quantize(x32, tok_o, ga)
    assert np.float32(gs.item()) == ga
    np.testing.assert_array_equal(q.cpu().numpy(), q_o)
    np.testing.assert_array_equal(sf.cpu().numpy(), sf_o)
    want_al = np.array([oracle.alpha(ga, g) for g in gs_w.numpy()], np.float32)
    np.testing.assert_array_equal(al.cpu().numpy(), want_al)


@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("T,H", [(33, 256), (512, 6144)])
def test_combine_within_bound(cuda_device, y_dtype, out_dtype, T, H):
    d = cuda_device
    E, k = 256, 8
    logits = workloads.normal(T, E, 1.0, 7000 + T)
    ex_o, _, w_o = oracle.route_topk(logits.numpy(), k)
    _, _, _, row_o = oracle.permute_by_expert(ex_o, E)
    w32 = w_o.astype(np.float32)
    y = workloads.normal(T * k, H, 1.0, 8000 + T).to(y_dtype)
    out = nv.moe_combine(y.to(d), torch.from_numpy(w32).to(d), torch.from_numpy(row_o.astype(np.int32)).to(d),
                         out_dtype=out_dtype)
    st, code = nv.last_device_error()
    assert st == 0, hex(code)
    y64 = y.to(torch.float64).numpy()
    v = oracle.combine(y64, w32.astype(np.float64), row_o)
    absum = oracle.combine(np.abs(y64), np.abs(w32.astype(np.float64)), row_o)
    half_ulp = {torch.float32: 0.0, torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}[out_dtype]
    bound = (k + 2) * 2.0 ** -24 * absum * (1 + half_ulp) + half_ulp * np.abs(v) + 1e-30
    got = out.to(torch.float64).cpu().numpy()
    err = np.abs(got - v)
    assert (err <= bound).all(), f"max err/bound {(err / bound).max():.3f}"
