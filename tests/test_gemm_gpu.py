"""GPU parity of the NVFP4 GEMM against the CPU oracle.

Tolerance (per element): |out - v| <= 2^-7 * |alpha| * sum_k |a_k b_k| + 1e-6, with v the
oracle's fp64 result. Bit-exact where the result is a single dequantised product (one-hot
rows, alpha = 1). Every config shape runs in the launch configuration the benchmark uses
(same planner, with split-K workspace); at sizes the oracle cannot finish in seconds, the
oracle computes sampled output rows and columns one by one."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle
from helpers import bf16_bits_of, check_within_tolerance, gpu_quantize

pytestmark = pytest.mark.gpu


def _oracle_operands(a, b, rows=None, cols=None):
    ga = oracle.global_scale(a.numpy())
    gb = oracle.global_scale(b.numpy())
    ar = a if rows is None else a[rows]
    br = b if cols is None else b[cols]
    qa, sa = oracle.quantize(ar.contiguous().numpy(), ga)
    qb, sb = oracle.quantize(br.contiguous().numpy(), gb)
    return qa, sa, qb, sb, oracle.alpha(ga, gb)


def run_case(dev, a, b, rows=None, cols=None, use_ws=True, guard=True, what=""):
    """CUDA path on the full problem; oracle on (optionally) sampled rows / columns."""
    M, K = a.shape
    N = b.shape[0]
    Aq, sfA, gsA = gpu_quantize(a, dev)
    Bq, sfB, gsB = gpu_quantize(b, dev)
    al = nv.alpha(gsA, gsB)
    ws = nv.make_workspace(M, N, K, dev) if use_ws else None
    pad = 3 if guard else 0
    sentinel = -12352.0   # exactly representable in bf16
    big = torch.full((M + pad, N), sentinel, dtype=torch.bfloat16, device=dev)
    out = big[:M]
    ws_guard = None
    if ws is not None and guard:
        ws_guard = torch.full((ws.numel() + 4096,), 0xA5, dtype=torch.uint8, device=dev)
        ws_guard[: ws.numel()] = 0
        ws = ws_guard[: ws.numel()]
    nv.gemm(Aq, sfA, Bq, sfB, al, out=out, workspace=ws)
    st, code = nv.last_device_error()
    assert st == 0, f"device error word {code:#x}"
    if guard and pad:
        assert (big[M:].float() == sentinel).all(), "write past the last output row"
    if ws_guard is not None:
        assert (ws_guard[ws.numel():] == 0xA5).all(), "write past the end of the workspace"
        # every tile counter is back to zero after a completed call
        assert int(ws_guard[:256].to(torch.int32).sum()) == 0
    qa, sa, qb, sb, alo = _oracle_operands(a, b, rows, cols)
    assert np.float32(al.item()) == alo
    v, S, _ = oracle.gemm(qa, sa, qb, sb, alo)
    o = out if rows is None else out[torch.as_tensor(rows, device=dev)]
    o = o if cols is None else o[:, torch.as_tensor(cols, device=dev)]
    check_within_tolerance(o, v, S, alo, what or f"{M}x{N}x{K}")
    return out


def _sample(n, k, seed):
    if n <= k:
        return None
    rng = np.random.default_rng(seed)
    idx = set(rng.choice(n, k - 4, replace=False).tolist()) | {0, 1, n - 2, n - 1}
    return np.array(sorted(idx))


def test_single_case_and_smoke_property(cuda_device):
    c = workloads.single_case()
    out = run_case(cuda_device, c.a(), c.b())
    # the reference page's smoke check on this shape: output not all zero, finite
    assert (out.float().abs() > 0).any() and torch.isfinite(out.float()).all()


@pytest.mark.parametrize("case", workloads.attn_proj_cases(), ids=lambda c: c.name)
def test_attn_proj_sweep(cuda_device, case):
    rows = _sample(case.M, 128, 1)
    run_case(cuda_device, case.a(), case.b(), rows=rows)


@pytest.mark.parametrize("case", workloads.moe_expert_cases(), ids=lambda c: c.name)
def test_moe_expert_sweep(cuda_device, case):
    rows = _sample(case.M, 96, 2)
    cols = _sample(case.N, 1024, 3) if case.M >= 512 else None
    run_case(cuda_device, case.a(), case.b(), rows=rows, cols=cols)


@pytest.mark.parametrize("case", workloads.plateau_cases(), ids=lambda c: c.name)
def test_plateau_sampled(cuda_device, case):
    rows = _sample(case.M, 48, 4)
    cols = _sample(case.N, 512, 5)
    run_case(cuda_device, case.a(), case.b(), rows=rows, cols=cols, guard=False)


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (17, 136, 512), (33, 8, 256), (64, 24, 768),
                                   (65, 264, 768), (130, 776, 1024), (200, 1032, 256),
                                   (129, 128, 2560), (300, 512, 4096), (16, 6144, 2048)])
def test_edge_shapes(cuda_device, M, N, K):
    a = workloads.normal(M, K, 1.0, M * 7 + N)
    b = workloads.normal(N, K, 0.02, N * 11 + K)
    run_case(cuda_device, a, b, use_ws=True)
    run_case(cuda_device, a, b, use_ws=False)


def test_zero_scales_give_exact_zero(cuda_device):
    a = torch.zeros(96, 512)
    b = workloads.normal(64, 512, 1.0, 3)
    for M in (16, 96):
        out = run_case(cuda_device, a[:M], b)
        assert (out.float() == 0).all()


def _one_hot_operands(M, K, seed):
    rng = np.random.default_rng(seed)
    ks = rng.integers(0, K, M)
    Aq = np.zeros((M, K // 2), np.uint8)
    for m, k in enumerate(ks):
        Aq[m, k // 2] = 0x2 << (4 * (k % 2))          # code 2 = 1.0
    sfA = np.full((M, K // 16), 0x38, np.uint8)        # scale 1.0
    return Aq, sfA


@pytest.mark.parametrize("M,N,K", [(16, 768, 6144), (64, 256, 512), (128, 256, 512),
                                   (300, 512, 1024)])
def test_one_hot_rows_bit_exact(cuda_device, M, N, K):
    Aq, sfA = _one_hot_operands(M, K, M + N)
    rng = np.random.default_rng(N)
    Bq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sfB = rng.integers(0x20, 0x50, (N, K // 16), dtype=np.uint8)
    v, S, _ = oracle.gemm(Aq, sfA, Bq, sfB, 1.0)
    want = oracle.bf16_bits(v)
    d = cuda_device
    alpha = torch.ones(1, device=d)
    for use_ws in (True, False):
        ws = nv.make_workspace(M, N, K, d) if use_ws else None
        out = nv.gemm(torch.from_numpy(Aq).to(d), torch.from_numpy(sfA).to(d),
                      torch.from_numpy(Bq).to(d), torch.from_numpy(sfB).to(d), alpha,
                      workspace=ws)
        np.testing.assert_array_equal(bf16_bits_of(out), want)


@pytest.mark.parametrize("cluster,groups", [(1, 1), (8, 1), (2, 6), (1, 12)])
def test_split_k_deterministic_and_within_tolerance(cuda_device, cluster, groups):
    c = workloads.attn_proj_cases()[0]          # M = 16: the most split-heavy shape
    with nv.plan_override(cluster=cluster, groups=groups):
        _split_k_deterministic(cuda_device, c, cluster, groups)


def _split_k_deterministic(cuda_device, c, cluster, groups):
    a, b = c.a(), c.b()
    d = cuda_device
    Aq, sfA, gsA = gpu_quantize(a, d)
    Bq, sfB, gsB = gpu_quantize(b, d)
    al = nv.alpha(gsA, gsB)
    assert (nv.gemm_workspace_size(c.M, c.N, c.K) > 0) == (groups > 1)
    ws = nv.make_workspace(c.M, c.N, c.K, d)
    o1 = nv.gemm(Aq, sfA, Bq, sfB, al, workspace=ws)
    o2 = nv.gemm(Aq, sfA, Bq, sfB, al, workspace=ws)
    assert torch.equal(bf16_bits_tensor(o1), bf16_bits_tensor(o2))
    qa, sa, qb, sb, alo = _oracle_operands(a, b)
    v, S, _ = oracle.gemm(qa, sa, qb, sb, alo)
    check_within_tolerance(o1, v, S, alo, f"split-K cluster={cluster} groups={groups}")


@pytest.mark.parametrize("cluster,groups", [(2, 1), (3, 1), (4, 1), (8, 1), (2, 3), (3, 2), (1, 5)])
@pytest.mark.parametrize("M,N,K", [(16, 768, 6144), (256, 768, 6144), (130, 776, 2560),
                                   (40, 264, 4096)])
def test_split_k_layouts(cuda_device, cluster, groups, M, N, K):
    """Every cluster / group layout of split-K (distributed-shared-memory reduction inside
    a cluster, workspace reduction across clusters) against the oracle."""
    a = workloads.normal(M, K, 1.0, M + 3 * N)
    b = workloads.normal(N, K, 0.02, N + 5 * K)
    with nv.plan_override(cluster=cluster, groups=groups):
        run_case(cuda_device, a, b, use_ws=True)


def bf16_bits_tensor(t):
    return t.view(torch.int16)


def test_transposed_product_agrees(cuda_device):
    a = workloads.normal(96, 1024, 1.0, 21)
    b = workloads.normal(40, 1024, 1.0, 22)
    d = cuda_device
    Aq, sfA, gsA = gpu_quantize(a, d)
    Bq, sfB, gsB = gpu_quantize(b, d)
    al = nv.alpha(gsA, gsB)
    o1 = nv.gemm(Aq, sfA, Bq, sfB, al, workspace=nv.make_workspace(96, 40, 1024, d))
    o2 = nv.gemm(Bq, sfB, Aq, sfA, al, workspace=nv.make_workspace(40, 96, 1024, d))
    qa, sa, qb, sb, alo = _oracle_operands(a, b)
    v, S, _ = oracle.gemm(qa, sa, qb, sb, alo)
    check_within_tolerance(o1, v, S, alo, "A B^T")
    check_within_tolerance(o2.t().contiguous(), v, S, alo, "(B A^T)^T")


def test_workspace_too_small_is_rejected(cuda_device):
    with nv.plan_override(cluster=2, groups=4):
        _workspace_too_small(cuda_device)


def _workspace_too_small(cuda_device):
    n = nv.gemm_workspace_size(16, 768, 6144)
    assert n > 0
    d = cuda_device
    ws = torch.zeros(n - 256, dtype=torch.uint8, device=d)
    Aq = torch.zeros(16, 3072, dtype=torch.uint8, device=d)
    sfA = torch.zeros(16, 384, dtype=torch.uint8, device=d)
    Bq = torch.zeros(768, 3072, dtype=torch.uint8, device=d)
    sfB = torch.zeros(768, 384, dtype=torch.uint8, device=d)
    with pytest.raises(nv.Nvfp4Error) as e:
        nv.gemm(Aq, sfA, Bq, sfB, torch.ones(1, device=d), workspace=ws)
    assert e.value.status == 7
