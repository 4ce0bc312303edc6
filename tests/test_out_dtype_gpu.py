"""GPU parity of the GEMMs' other output types (the mm_fp4 signature's out_dtype: "The Art of
Reading the Manual", section "The Message"): fp16 and fp32 beside the default bf16.

The kernel computes alpha * acc in fp32 and rounds it once to the output type. Where the
result is one exact dequantised product (one-hot rows, alpha a power of two) that equals the
oracle's single rounding of its fp64 value, so those rows are compared bit for bit: fp16
against oracle.fp16_bits (overflow to infinity included), fp32 against numpy's fp64 -> fp32
conversion. Everywhere else the GEMM tolerance 2^-7 |alpha| sum|a b| + 1e-6 applies, on every
epilogue path: row stores (non-swap tiles), per-token stores (few-token and grouped tiles),
the split-K reductions inside a cluster and through the workspace, both scale layouts."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle
from helpers import check_within_tolerance, gpu_quantize, tile_np

pytestmark = pytest.mark.gpu

DTYPES = [torch.float16, torch.float32]


def _bits(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.float32:
        return t.contiguous().view(torch.int32).cpu().numpy().view(np.uint32)
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _want_bits(v: np.ndarray, dtype) -> np.ndarray:
    if dtype == torch.float32:
        return v.astype(np.float32).view(np.uint32)
    return oracle.fp16_bits(v)


def _one_hot_operands(M, K, seed):
    rng = np.random.default_rng(seed)
    ks = rng.integers(0, K, M)
    Aq = np.zeros((M, K // 2), np.uint8)
    for m, k in enumerate(ks):
        Aq[m, k // 2] = 0x2 << (4 * (k % 2))          # code 2 = 1.0
    sfA = np.full((M, K // 16), 0x38, np.uint8)        # scale 1.0
    return Aq, sfA


@pytest.mark.parametrize("dtype", DTYPES, ids=str)
@pytest.mark.parametrize("alpha", [1.0, 2048.0])
@pytest.mark.parametrize("M,N,K", [(16, 768, 6144), (64, 256, 512), (300, 512, 1024), (130, 1024, 2048)])
def test_one_hot_rows_bit_exact(cuda_device, dtype, alpha, M, N, K):
    """One exact product per output: bit-identical to the oracle's rounding; with alpha =
    2048 many fp16 results exceed 65504 and must be infinity."""
    Aq, sfA = _one_hot_operands(M, K, M + N)
    rng = np.random.default_rng(N)
    Bq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sfB = rng.integers(0x20, 0x50, (N, K // 16), dtype=np.uint8)
    v, S, _ = oracle.gemm(Aq, sfA, Bq, sfB, alpha)
    want = _want_bits(v, dtype)
    if dtype == torch.float16 and alpha > 1:
        assert (want == 0x7C00).any() and (want == 0xFC00).any(), "the case must overflow fp16"
    d = cuda_device
    al = torch.full((1,), alpha, device=d)
    for tiled in (False, True):
        for use_ws in (True, False):
            A_t, B_t = torch.from_numpy(Aq).to(d), torch.from_numpy(Bq).to(d)
            sA = torch.from_numpy(tile_np(sfA, K) if tiled else sfA).to(d)
            sB = torch.from_numpy(tile_np(sfB, K) if tiled else sfB).to(d)
            ws = nv.make_workspace(M, N, K, d) if use_ws else None
            out = nv.gemm(A_t, sA, B_t, sB, al, workspace=ws, tiled=tiled, out_dtype=dtype)
            assert out.dtype == dtype
            np.testing.assert_array_equal(_bits(out), want, err_msg=f"tiled={tiled} ws={use_ws}")


def _run(dev, a, b, dtype, tiled=False, rows=None, cols=None):
    M, K = a.shape
    N = b.shape[0]
    Aq, sfA, gsA = gpu_quantize(a, dev)
    Bq, sfB, gsB = gpu_quantize(b, dev)
    al = nv.alpha(gsA, gsB)
    if tiled:
        sfA, sfB = nv.sf_tile(sfA), nv.sf_tile(sfB)
    sentinel = -12352.0
    big = torch.full((M + 2, N), sentinel, dtype=dtype, device=dev)
    out = big[:M]
    nv.gemm(Aq, sfA, Bq, sfB, al, out=out, workspace=nv.make_workspace(M, N, K, dev), tiled=tiled)
    st, code = nv.last_device_error()
    assert st == 0, hex(code)
    assert (big[M:].float() == sentinel).all(), "write past the last output row"
    ga, gb = oracle.global_scale(a.numpy()), oracle.global_scale(b.numpy())
    ar = a if rows is None else a[rows]
    br = b if cols is None else b[cols]
    qa, sa = oracle.quantize(ar.contiguous().numpy(), ga)
    qb, sb = oracle.quantize(br.contiguous().numpy(), gb)
    alo = oracle.alpha(ga, gb)
    v, S, _ = oracle.gemm(qa, sa, qb, sb, alo)
    o = out if rows is None else out[torch.as_tensor(rows, device=dev)]
    o = o if cols is None else o[:, torch.as_tensor(cols, device=dev)]
    check_within_tolerance(o, v, S, alo, f"{M}x{N}x{K} {dtype} tiled={tiled}")


@pytest.mark.parametrize("dtype", DTYPES, ids=str)
@pytest.mark.parametrize("case", [workloads.single_case()] + workloads.attn_proj_cases(),
                         ids=lambda c: c.name)
def test_config_shapes_within_tolerance(cuda_device, dtype, case):
    rows = None if case.M <= 256 else np.r_[0:64, case.M - 64:case.M]
    for tiled in (False, True):
        _run(cuda_device, case.a(), case.b(), dtype, tiled=tiled, rows=rows)


@pytest.mark.parametrize("dtype", DTYPES, ids=str)
@pytest.mark.parametrize("M,N,K", [(40, 264, 4096), (130, 776, 2560), (17, 136, 512), (200, 1032, 256)])
def test_ragged_shapes(cuda_device, dtype, M, N, K):
    a = workloads.normal(M, K, 1.0, M * 7 + N)
    b = workloads.normal(N, K, 0.02, N * 11 + K)
    _run(cuda_device, a, b, dtype)


@pytest.mark.parametrize("dtype", DTYPES, ids=str)
@pytest.mark.parametrize("cluster,groups", [(4, 1), (2, 3)])
def test_split_k_reductions(cuda_device, dtype, cluster, groups):
    """The reduced chunk stores of split-K: inside one cluster, and across clusters through the
    workspace."""
    for M, N, K in ((16, 768, 6144), (256, 768, 6144)):
        a = workloads.normal(M, K, 1.0, M + 1)
        b = workloads.normal(N, K, 0.02, N + 2)
        with nv.plan_override(cluster=cluster, groups=groups):
            _run(cuda_device, a, b, dtype)


@pytest.mark.parametrize("dtype", DTYPES, ids=str)
def test_plateau_4096_sampled(cuda_device, dtype):
    c = workloads.plateau_cases()[0]
    rng = np.random.default_rng(9)
    rows = np.sort(rng.choice(c.M, 32, replace=False))
    cols = np.sort(rng.choice(c.N, 256, replace=False))
    _run(cuda_device, c.a(), c.b(), dtype, tiled=True, rows=rows, cols=cols)


@pytest.mark.parametrize("dtype", DTYPES, ids=str)
def test_grouped_out_dtype(cuda_device, dtype):
    d = cuda_device
    counts = [5, 0, 37, 20, 130]
    E, N, K = len(counts), 256, 512
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(off[-1])
    a = workloads.normal(rows, K, 1.0, 41)
    bs = [workloads.normal(N, K, 0.02, 50 + e) for e in range(E)]
    ad = a.to(d)
    gsA = nv.global_scale(ad)
    Aq, sfA = nv.quantize(ad, gsA)
    Bq = torch.empty(E, N, K // 2, dtype=torch.uint8, device=d)
    sfB = torch.empty(E, N, K // 16, dtype=torch.uint8, device=d)
    gsB = torch.empty(E, dtype=torch.float32, device=d)
    for e in range(E):
        bd = bs[e].to(d)
        nv.global_scale(bd, out=gsB[e:e + 1])
        nv.quantize(bd, gsB[e:e + 1], q=Bq[e], sf=sfB[e])
    al = nv.alpha(gsA, gsB)
    out = torch.full((rows + 3, N), 777.0, dtype=dtype, device=d)
    offs = torch.from_numpy(off).to(d)
    nv.grouped_gemm(Aq, sfA, Bq, sfB, al, offs, out=out[:rows])
    st, code = nv.last_device_error()
    assert st == 0, hex(code)
    assert (out[rows:].float() == 777.0).all()
    ga = oracle.global_scale(a.numpy())
    qa, sa = oracle.quantize(a.numpy(), ga)
    parts = [oracle.quantize(b.numpy(), oracle.global_scale(b.numpy())) for b in bs]
    alo = np.array([oracle.alpha(ga, oracle.global_scale(b.numpy())) for b in bs], np.float32)
    v, S, _ = oracle.grouped_gemm(qa, sa, np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]),
                                  alo, off)
    for e in range(E):
        r0, r1 = off[e], off[e + 1]
        if r1 > r0:
            check_within_tolerance(out[r0:r1], v[r0:r1], S[r0:r1], alo[e], f"expert {e} {dtype}")


def test_bad_out_dtype_is_rejected(cuda_device):
    lib = nv.load()
    st = lib.nvfp4_gemm_ex2(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 16, 768, 6144, None, 0, 0, 3, None)
    assert st == 1
    with pytest.raises(ValueError):
        nv.gemm(torch.zeros(16, 256, dtype=torch.uint8, device=cuda_device),
                torch.zeros(16, 32, dtype=torch.uint8, device=cuda_device),
                torch.zeros(8, 256, dtype=torch.uint8, device=cuda_device),
                torch.zeros(8, 32, dtype=torch.uint8, device=cuda_device),
                torch.ones(1, device=cuda_device), out_dtype=torch.int32)
