"""GPU checks of the grouped (mixture-of-experts) GEMM run as CTA pairs: the two CTAs of a
2-CTA cluster hold 128 weight rows each of a 256-row pair of one expert and half of the
expert's token tile, and the 2-SM MMA (tcgen05.mma.cta_group::2) reads both.

Every output element is the same sequence of 64-wide block-scaled products as in the
single-CTA grouped launch, so the two must agree bit for bit; both are within the GEMM
tolerance of the CPU oracle. Cases: ragged and empty experts, token tiles of 128 and 176 rows,
a weight count that ends inside a pair (N = 264: the last pair's second tile is all past N),
rows past the last expert left untouched, and the T = 4096 MoE densities at full size."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle
from helpers import check_within_tolerance

pytestmark = pytest.mark.gpu

SENTINEL = 776.0   # exactly representable in bf16


def _operands(dev, counts, N, K, seed):
    E = len(counts)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(off[-1])
    a = workloads.normal(max(rows, 1), K, 1.0, seed)[:rows]
    bs = [workloads.normal(N, K, 0.02, seed + 100 + e) for e in range(E)]
    ad = a.to(dev)
    gsA = nv.global_scale(ad)
    Aq, sfA = nv.quantize(ad, gsA)
    Bq = torch.empty(E, N, K // 2, dtype=torch.uint8, device=dev)
    sfB = torch.empty(E, N, K // 16, dtype=torch.uint8, device=dev)
    gsB = torch.empty(E, dtype=torch.float32, device=dev)
    for e in range(E):
        bd = bs[e].to(dev)
        nv.global_scale(bd, out=gsB[e:e + 1])
        nv.quantize(bd, gsB[e:e + 1], q=Bq[e], sf=sfB[e])
    al = nv.alpha(gsA, gsB)
    return a, bs, off, (Aq, sfA, Bq, sfB, al, torch.from_numpy(off).to(dev))


def _run(ops, rows, N, pad_rows, pair, grouped_bn):
    Aq, sfA, Bq, sfB, al, off = ops
    out = torch.full((rows + pad_rows, N), SENTINEL, dtype=torch.bfloat16, device=Aq.device)
    with nv.plan_override(grouped_bn=grouped_bn, pair=pair):
        nv.grouped_gemm(Aq, sfA, Bq, sfB, al, off, out=out[:rows] if pad_rows else out)
    st, code = nv.last_device_error()
    assert st == 0, hex(code)
    if pad_rows:
        assert (out[rows:].float() == SENTINEL).all(), "write past the last expert's rows"
    return out[:rows]


@pytest.mark.parametrize("grouped_bn", [128, 176])
@pytest.mark.parametrize("N", [512, 264])
def test_grouped_pair_matches_single_cta_and_oracle(cuda_device, grouped_bn, N):
    d = cuda_device
    K = 1024
    counts = [0, 1, 177, 90, 3, 150, 0, 33, 128]
    a, bs, off, ops = _operands(d, counts, N, K, 70 + grouped_bn + N)
    rows = int(off[-1])
    o_pair = _run(ops, rows, N, 4, pair=2, grouped_bn=grouped_bn)
    o_single = _run(ops, rows, N, 4, pair=1, grouped_bn=grouped_bn)
    assert torch.equal(o_pair.view(torch.int16), o_single.view(torch.int16)), "pair != single-CTA tiles"
    ga = oracle.global_scale(a.numpy())
    qa, sa = oracle.quantize(a.numpy(), ga)
    for e in range(len(counts)):
        r0, r1 = int(off[e]), int(off[e + 1])
        if r1 == r0:
            continue
        gb = oracle.global_scale(bs[e].numpy())
        qb, sb = oracle.quantize(bs[e].numpy(), gb)
        alo = oracle.alpha(ga, gb)
        v, S, _ = oracle.gemm(qa[r0:r1], sa[r0:r1], qb, sb, alo)
        check_within_tolerance(o_pair[r0:r1], v, S, alo, f"pair expert {e}")


@pytest.mark.parametrize("name", ["moe_down_T4096", "moe_gate_up_T4096"])
def test_grouped_pair_full_density(cuda_device, name):
    """The T = 4096 MoE GEMMs (256 experts, 99-168 rows each) at full size: pairs give the
    same bits as the single-CTA launch."""
    d = cuda_device
    case = [c for c in workloads.grouped_cases() if c.name == name][0]
    r = case.route()
    a = case.a(r.rows)
    ad = a.to(d)
    gsA = nv.global_scale(ad)
    Aq, sfA = nv.quantize(ad, gsA)
    del ad
    E, N, K = case.num_experts, case.N, case.K
    Bq = torch.empty(E, N, K // 2, dtype=torch.uint8, device=d)
    sfB = torch.empty(E, N, K // 16, dtype=torch.uint8, device=d)
    gsB = torch.empty(E, dtype=torch.float32, device=d)
    for e in range(E):
        bd = case.b(e, d)
        nv.global_scale(bd, out=gsB[e:e + 1])
        nv.quantize(bd, gsB[e:e + 1], q=Bq[e], sf=sfB[e])
    al = nv.alpha(gsA, gsB)
    off = r.offsets.to(d)
    outs = []
    for pair in (2, 1):
        with nv.plan_override(pair=pair):
            outs.append(nv.grouped_gemm(Aq, sfA, Bq, sfB, al, off))
        st, code = nv.last_device_error()
        assert st == 0, hex(code)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16)), name


@pytest.mark.parametrize("grouped_bn", [128, 176])
def test_grouped_pair_swiglu_matches_single_cta(cuda_device, grouped_bn):
    """The gate_up GEMM with the fused SwiGLU + NVFP4 epilogue: each CTA of a pair holds its
    own 64 gate rows and the 64 matching up rows, so h's codes and block scales are the same
    bytes with and without pairs (rows past the last expert untouched)."""
    d = cuda_device
    K, I = 1024, 256
    counts = [130, 0, 177, 95, 1, 160, 128]
    _, _, off, ops = _operands(d, counts, 2 * I, K, 90 + grouped_bn)
    Aq, sfA, Bq, sfB, al, offd = ops
    rows = int(off[-1])
    gs_h = torch.full((1,), 64.0, dtype=torch.float32, device=d)
    res = []
    for pair in (2, 1):
        hq = torch.full((rows + 3, I // 2), 0xA7, dtype=torch.uint8, device=d)
        hsf = torch.full((rows + 3, I // 16), 0xA7, dtype=torch.uint8, device=d)
        with nv.plan_override(grouped_bn=grouped_bn, pair=pair):
            nv.grouped_gemm_swiglu(Aq, sfA, Bq, sfB, al, offd, gs_h, h_q=hq[:rows], h_sf=hsf[:rows])
        st, code = nv.last_device_error()
        assert st == 0, hex(code)
        assert (hq[rows:] == 0xA7).all() and (hsf[rows:] == 0xA7).all(), "write past the rows"
        res.append((hq[:rows].clone(), hsf[:rows].clone()))
    assert torch.equal(res[0][0], res[1][0]), "h codes differ with pairs"
    assert torch.equal(res[0][1], res[1][1]), "h scales differ with pairs"


@pytest.mark.parametrize("out_dtype", [torch.float16, torch.float32])
def test_grouped_pair_output_dtypes(cuda_device, out_dtype):
    """fp16 and fp32 outputs of the grouped pairs: the same bits as the single-CTA launch."""
    d = cuda_device
    counts = [140, 3, 0, 176, 99]
    _, _, off, ops = _operands(d, counts, 384, 512, 130)
    Aq, sfA, Bq, sfB, al, offd = ops
    outs = []
    for pair in (2, 1):
        with nv.plan_override(grouped_bn=176, pair=pair):
            outs.append(nv.grouped_gemm(Aq, sfA, Bq, sfB, al, offd, out_dtype=out_dtype))
        st, code = nv.last_device_error()
        assert st == 0, hex(code)
    view = torch.int16 if out_dtype == torch.float16 else torch.int32
    assert torch.equal(outs[0].view(view), outs[1].view(view))
