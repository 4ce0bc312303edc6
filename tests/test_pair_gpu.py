"""GPU checks of the CTA-pair launch of the dense GEMM: the two CTAs of a 2-CTA cluster compute
one 256 x 256 (or, on request, 256 x 128) tile with the 2-SM MMA (tcgen05.mma.cta_group::2): each
loads its own 128 rows of the token tile and its half of the weight tile, and the even CTA's MMAs
read both CTAs' shared memory.

Every output element is the same sequence of 64-wide block-scaled products with or without
pairs, so the two launches must agree bit for bit; both must be within the GEMM tolerance of
the CPU oracle (2^-7 |alpha| sum|a b| + 1e-6). Shapes cover an odd number of row tiles (the
last pair's second CTA has no rows), weight rows that end inside a tile's second half (that
half reads as zero), NVFP4 and MXFP4, and the plateau shapes. (The planner uses pairs wherever
they apply; the plan override switches them off for the comparison.)"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle
from helpers import check_within_tolerance, gpu_quantize

pytestmark = pytest.mark.gpu


def _operands(dev, a, b):
    Aq, sfA, gsA = gpu_quantize(a, dev)
    Bq, sfB, gsB = gpu_quantize(b, dev)
    return Aq, nv.sf_tile(sfA), Bq, nv.sf_tile(sfB), nv.alpha(gsA, gsB)


def _gemm(Aq, sA, Bq, sB, al, M, N, pair, bn=256):
    out = torch.full((M + 2, N), -12352.0, dtype=torch.bfloat16, device=Aq.device)
    with nv.plan_override(bn=bn, cluster=1, groups=1, pair=pair):
        nv.gemm(Aq, sA, Bq, sB, al, out=out[:M], tiled=True)
    st, code = nv.last_device_error()
    assert st == 0, hex(code)
    assert (out[M:].float() == -12352.0).all(), "write past the last output row"
    return out[:M]


@pytest.mark.parametrize("bn", [256, 128])
@pytest.mark.parametrize("M,N,K", [(300, 776, 1024), (512, 1024, 2048), (1000, 264, 512),
                                   (129, 520, 768), (256, 256, 256), (640, 2048, 6144)])
def test_pair_matches_single_cta_and_oracle(cuda_device, M, N, K, bn):
    d = cuda_device
    a = workloads.normal(M, K, 1.0, 3 * M + N)
    b = workloads.normal(N, K, 0.02, 5 * N + K)
    ops = _operands(d, a, b)
    o_pair = _gemm(*ops, M, N, pair=2, bn=bn)
    o_single = _gemm(*ops, M, N, pair=1, bn=bn)
    assert torch.equal(o_pair.view(torch.int16), o_single.view(torch.int16)), "pair != single-CTA tiles"
    ga, gb = oracle.global_scale(a.numpy()), oracle.global_scale(b.numpy())
    rows = np.r_[0:min(M, 40), max(0, M - 40):M]
    qa, sa = oracle.quantize(a[rows].contiguous().numpy(), ga)
    qb, sb = oracle.quantize(b.numpy(), gb)
    alo = oracle.alpha(ga, gb)
    v, S, _ = oracle.gemm(qa, sa, qb, sb, alo)
    check_within_tolerance(o_pair[torch.as_tensor(rows, device=d)], v, S, alo, f"pair {M}x{N}x{K}")


@pytest.mark.parametrize("bn", [256, 128])
@pytest.mark.parametrize("M,N,K", [(300, 776, 1024), (512, 1024, 2048)])
def test_pair_mx(cuda_device, M, N, K, bn):
    d = cuda_device
    a = workloads.normal(M, K, 1.0, 7 * M + N)
    b = workloads.normal(N, K, 0.02, 9 * N + K)
    qa, sa = nv.mx_quantize(a.to(d), tiled=True)
    qb, sb = nv.mx_quantize(b.to(d), tiled=True)
    al = torch.ones(1, device=d)
    outs = []
    for pair in (2, 1):
        with nv.plan_override(bn=bn, cluster=1, groups=1, pair=pair):
            outs.append(nv.mx_gemm(qa, sa, qb, sb, al))
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    qa_o, sa_o = oracle.mx_quantize(a.numpy())
    qb_o, sb_o = oracle.mx_quantize(b.numpy())
    v, S, _ = oracle.mx_gemm(qa_o, sa_o, qb_o, sb_o, 1.0)
    check_within_tolerance(outs[0], v, S, 1.0, f"mx pair {M}x{N}x{K}")


def test_pairs_on_the_plateau(cuda_device):
    """4096^3 and 8192^3 with tiled scales: the default plan (pairs) gives the same bits as
    single-CTA tiles."""
    d = cuda_device
    for c in workloads.plateau_cases()[:2]:
        ops = _operands(d, c.a(), c.b())
        o_default = nv.gemm(*ops, tiled=True)
        with nv.plan_override(pair=1):
            o_single = nv.gemm(*ops, tiled=True)
        assert torch.equal(o_default.view(torch.int16), o_single.view(torch.int16)), c.name


@pytest.mark.parametrize("M,N,K", [(2500, 2056, 1024), (4096, 4096, 3072)])
def test_pair_half_tiles(cuda_device, M, N, K):
    """A last wave of 256 x 256 pair tiles that fills at most half of the pairs runs as
    256 x 128 halves. On 148 SMs (74 pairs): 2500 x 2056 has 10 x 9 = 90 tiles, the last 16
    split in halves, the last Q tile 8 columns wide (its second half starts past N) and the
    last P tile 68 rows; 4096 x 4096 has 256 tiles, the last 34 split. Same bits as the
    single-CTA tiles and as pairs without halves, within tolerance of the oracle."""
    d = cuda_device
    a = workloads.normal(M, K, 1.0, 11 * M + N)
    b = workloads.normal(N, K, 0.02, 13 * N + K)
    ops = _operands(d, a, b)
    o_half = _gemm(*ops, M, N, pair=2)
    o_whole = _gemm(*ops, M, N, pair=3) if K >= 3072 else None
    o_single = _gemm(*ops, M, N, pair=1)
    assert torch.equal(o_half.view(torch.int16), o_single.view(torch.int16)), "half tiles != single-CTA tiles"
    if o_whole is not None:
        assert torch.equal(o_half.view(torch.int16), o_whole.view(torch.int16)), "half tiles != whole pair tiles"
    ga, gb = oracle.global_scale(a.numpy()), oracle.global_scale(b.numpy())
    rows = np.r_[0:24, M - 72:M]
    qa, sa = oracle.quantize(a[rows].contiguous().numpy(), ga)
    qb, sb = oracle.quantize(b.numpy(), gb)
    alo = oracle.alpha(ga, gb)
    v, S, _ = oracle.gemm(qa, sa, qb, sb, alo)
    check_within_tolerance(o_half[torch.as_tensor(rows, device=d)], v, S, alo, f"half tiles {M}x{N}x{K}")


def test_pair_half_tiles_mx(cuda_device):
    d = cuda_device
    M, N, K = 2500, 2056, 1024
    a = workloads.normal(M, K, 1.0, 17 * M + N)
    b = workloads.normal(N, K, 0.02, 19 * N + K)
    qa, sa = nv.mx_quantize(a.to(d), tiled=True)
    qb, sb = nv.mx_quantize(b.to(d), tiled=True)
    al = torch.ones(1, device=d)
    outs = []
    for pair in (2, 1):
        with nv.plan_override(bn=256, cluster=1, groups=1, pair=pair):
            outs.append(nv.mx_gemm(qa, sa, qb, sb, al))
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    rows = np.r_[0:16, M - 48:M]
    qa_o, sa_o = oracle.mx_quantize(a[rows].contiguous().numpy())
    qb_o, sb_o = oracle.mx_quantize(b.numpy())
    v, S, _ = oracle.mx_gemm(qa_o, sa_o, qb_o, sb_o, 1.0)
    check_within_tolerance(outs[0][torch.as_tensor(rows, device=d)], v, S, 1.0, f"mx half tiles {M}x{N}x{K}")


@pytest.mark.parametrize("out_dtype", [torch.float16, torch.float32])
def test_pair_half_tiles_output_dtypes(cuda_device, out_dtype):
    """fp16 and fp32 outputs of pair tiles and of the half tiles of a short last wave
    (4096 x 4096 x 3072: 256 pair tiles on 74 pairs, the last 34 split): the same bits as
    single-CTA tiles."""
    d = cuda_device
    M, N, K = 4096, 4096, 3072
    a = workloads.normal(M, K, 1.0, 41)
    b = workloads.normal(N, K, 0.02, 43)
    Aq, sA, Bq, sB, al = _operands(d, a, b)
    outs = []
    for pair in (0, 1):
        with nv.plan_override(pair=pair):
            outs.append(nv.gemm(Aq, sA, Bq, sB, al, tiled=True, out_dtype=out_dtype))
        st, code = nv.last_device_error()
        assert st == 0, hex(code)
    view = torch.int16 if out_dtype == torch.float16 else torch.int32
    assert torch.equal(outs[0].view(view), outs[1].view(view))
