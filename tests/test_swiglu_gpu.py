"""GPU parity of the grouped gate_up GEMM with the fused SwiGLU + NVFP4 epilogue
(nvfp4_grouped_gemm_swiglu) against the CPU oracle (oracle.grouped_gemm, oracle.swiglu,
oracle.swiglu_quantize): the MoE expert MLP of "When a Benchmark Crashes", section "Why This
Message Was Written" (256 experts, intermediate size 2048).

Two kinds of checks:

* Bit-exact pin. With one-hot activation rows the gate / up values are single dequantised
  products, and with every gate value >= 24 silu(g) = g / (1 + exp(-g)) rounds to g in fp32
  (exp(-24) < 2^-34) and to within 4e-11 of g in fp64, so h = g u is exact on both sides and
  the quantised bytes (codes and scales) must equal the oracle's for every token-tile width.
  A gate / up row mix-up, a wrong block index or nibble order changes them.
* Full MoE configs (T = 512 and 4096 tokens, K = 6144, I = 2048), sampled experts and blocks.
  The kernel evaluates h in fp32 from its fp32 accumulators with CUDA's expf, the oracle in
  fp64 from the exact products, so a code may differ next to a rounding boundary. Bound per
  element, derived from the GEMM tolerance tol = 2^-7 |alpha| S + 1e-6 of g and u, silu's
  Lipschitz constant (|silu'| <= 1.0999) and NVFP4's rounding (half a code step, at most one
  unit of the block scale, plus the e4m3 rounding of the scale itself, at most 1/16 of it,
  times the 6 of the largest code, and 6 * 2^-10 below the e4m3 range):
      |deq_gpu - h_ref| <= E_h + E_q,
      E_h = 1.1 |u| tol_g + |silu(g)| tol_u + tol_g tol_u + 2^-21 |h_ref|,
      E_q = (1.5 s_gpu + 6 * 2^-10) / gs_h,   s_gpu the kernel's decoded block scale;
  and code equality wherever the kernel's block scale equals the oracle's and the oracle's
  scaled value y = h r lies farther than E'_h r from every e2m1 rounding boundary, where E'_h is
  E_h with tol replaced by the worst-case error of an fp32 sum of K terms in any order plus the
  alpha multiply, (K + 1) 2^-24 |alpha| S (the kernel's accumulator is fp32). Overall at least
  99% of the sampled codes and 98% of the block scales agree.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle

pytestmark = pytest.mark.gpu

E2M1_BOUNDARIES = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
SENTINEL = 0xA7


def _codes(q: np.ndarray) -> np.ndarray:
    """Packed bytes [rows, n/2] -> codes [rows, n] (element 2i in the low nibble)."""
    out = np.empty((q.shape[0], q.shape[1] * 2), np.uint8)
    out[:, 0::2] = q & 0xF
    out[:, 1::2] = q >> 4
    return out


def _run_gpu(dev, Aq, sfA, Bq, sfB, alphas, off, gs_h, rows_total, pad=3):
    I = Bq.shape[1] // 2
    hq = torch.full((rows_total + pad, I // 2), SENTINEL, dtype=torch.uint8, device=dev)
    hsf = torch.full((rows_total + pad, I // 16), SENTINEL, dtype=torch.uint8, device=dev)
    nv.grouped_gemm_swiglu(Aq, sfA, Bq, sfB, alphas, off, gs_h, h_q=hq[:rows_total], h_sf=hsf[:rows_total])
    st, code = nv.last_device_error()
    assert st == 0, hex(code)
    assert (hq[rows_total:] == SENTINEL).all() and (hsf[rows_total:] == SENTINEL).all(), "write past the rows"
    return hq[:rows_total].cpu().numpy(), hsf[:rows_total].cpu().numpy()


@pytest.mark.parametrize("grouped_bn", [32, 64, 128, 176, 256])
def test_swiglu_bit_exact_on_exact_products(cuda_device, grouped_bn):
    d = cuda_device
    rng = np.random.default_rng(7 + grouped_bn)
    counts = [5, 0, 37, 20, 70, 1]
    E, I, K = len(counts), 128, 512
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(off[-1]) + 4                            # 4 rows past the last expert
    ks = rng.integers(0, K, rows)
    Aq = np.zeros((rows, K // 2), np.uint8)
    for r, k in enumerate(ks):
        Aq[r, k // 2] = 0x2 << (4 * (k % 2))           # code 2 = 1.0
    sfA = np.full((rows, K // 16), 0x38, np.uint8)     # scale 1.0
    Bq = np.empty((E, 2 * I, K // 2), np.uint8)
    sfB = np.empty((E, 2 * I, K // 16), np.uint8)
    Bq[:, :I] = 0x77                                   # gate codes 7: value 6
    sfB[:, :I] = rng.choice(np.array([0x48, 0x50, 0x58], np.uint8), (E, I, K // 16))   # 4, 8, 16
    Bq[:, I:] = rng.integers(0, 256, (E, I, K // 2), dtype=np.uint8)
    sfB[:, I:] = rng.integers(0x20, 0x50, (E, I, K // 16), dtype=np.uint8)
    alphas = np.ones(E, np.float32)
    v, S, _ = oracle.grouped_gemm(Aq, sfA, Bq, sfB, alphas, off)
    used = int(off[-1])
    h = oracle.swiglu(v[:used])
    gs_h = np.float32(2688.0 / np.abs(h).max())
    q_ref, sf_ref, h32 = oracle.swiglu_quantize(v[:used], gs_h)
    assert np.array_equal(h32, (v[:used, :I] * v[:used, I:]).astype(np.float32)), "exact-product premise"
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(d)
    with nv.plan_override(grouped_bn=grouped_bn):
        hq, hsf = _run_gpu(d, t(Aq), t(sfA), t(Bq), t(sfB), t(alphas), t(off), t(np.array([gs_h])), rows)
    np.testing.assert_array_equal(hsf[:used], sf_ref)
    np.testing.assert_array_equal(hq[:used], q_ref)
    # rows of A past the last expert are not output rows of any expert: untouched
    assert (hq[used:] == SENTINEL).all() and (hsf[used:] == SENTINEL).all()


def _check_sampled(hq_e, hsf_e, v_g, v_u, S_g, S_u, alpha, gs_h, blocks, K, what):
    """Property checks of one expert's rows on the sampled blocks (v_g, v_u: [rows, 16 nb])."""
    nb = len(blocks)
    q_gpu = np.concatenate([hq_e[:, b * 8:(b + 1) * 8] for b in blocks], axis=1)
    sf_gpu = hsf_e[:, blocks]
    v = np.concatenate([v_g, v_u], axis=1)
    q_ref, sf_ref, h32 = oracle.swiglu_quantize(v, gs_h)
    h_ref = oracle.swiglu(v)
    deq = oracle.dequantize(q_gpu, sf_gpu) / float(gs_h)
    tol_g = oracle.tolerance(S_g, alpha)
    tol_u = oracle.tolerance(S_u, alpha)
    silu_g = oracle.silu(v_g)
    e_h = 1.1 * np.abs(v_u) * tol_g + np.abs(silu_g) * tol_u + tol_g * tol_u + 2.0 ** -21 * np.abs(h_ref)
    s_gpu = np.array([[oracle.e4m3_decode(int(x)) for x in row] for row in sf_gpu])
    e_q = np.repeat((1.5 * s_gpu + 6 * 2.0 ** -10) / float(gs_h), 16, axis=1)
    err = np.abs(deq - h_ref)
    bad = err > e_h + e_q
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} elements beyond the bound, e.g. "
                           f"{[(tuple(i), deq[tuple(i)], h_ref[tuple(i)], (e_h + e_q)[tuple(i)]) for i in np.argwhere(bad)[:4]]}")
    # scales: equal except where the block maximum sits next to an e4m3 rounding boundary
    same = sf_gpu == sf_ref
    assert same.mean() >= 0.98, f"{what}: only {same.mean():.3f} of the block scales agree"
    # codes: equal wherever the scale agrees and y is clear of every rounding boundary
    sfd_ref = np.array([[oracle.e4m3_decode(int(x)) for x in row] for row in sf_ref], np.float32)
    with np.errstate(divide="ignore"):
        r_ref = np.where(sfd_ref == 0, np.float32(0), np.float32(gs_h) / sfd_ref).astype(np.float32)
    y = h32 * np.repeat(r_ref, 16, axis=1)
    acc_g = (K + 1) * 2.0 ** -24 * abs(float(alpha)) * S_g
    acc_u = (K + 1) * 2.0 ** -24 * abs(float(alpha)) * S_u
    e_h32 = 1.1 * np.abs(v_u) * acc_g + np.abs(silu_g) * acc_u + acc_g * acc_u + 2.0 ** -21 * np.abs(h_ref)
    margin = e_h32 * np.repeat(r_ref, 16, axis=1) * 1.01 + 2.0 ** -20 * np.abs(y)
    ay = np.abs(y)
    clear = (np.min(np.abs(ay[..., None] - E2M1_BOUNDARIES), axis=-1) > margin) & (ay > margin)
    clear &= np.repeat(same, 16, axis=1)
    c_gpu, c_ref = _codes(q_gpu), _codes(q_ref)
    diff = clear & (c_gpu != c_ref)
    assert not diff.any(), f"{what}: {int(diff.sum())} codes differ away from rounding boundaries"
    assert clear.mean() > 0.5, f"{what}: too few elements clear of the boundaries ({clear.mean():.3f})"
    agree = (c_gpu == c_ref).mean()
    assert agree >= 0.99, f"{what}: only {agree:.4f} of the codes agree"
    return nb


@pytest.mark.parametrize("case", [c for c in workloads.grouped_cases() if "gate_up" in c.name],
                         ids=lambda c: c.name)
def test_swiglu_full_configs_sampled(cuda_device, case):
    d = cuda_device
    r = case.route()
    rows = r.rows
    a = case.a(rows)
    ad = a.to(d)
    gsA = nv.global_scale(ad)
    Aq, sfA = nv.quantize(ad, gsA)
    del ad
    E, N, K = case.num_experts, case.N, case.K
    I = N // 2
    Bq = torch.empty(E, N, K // 2, dtype=torch.uint8, device=d)
    sfB = torch.empty(E, N, K // 16, dtype=torch.uint8, device=d)
    gsB = torch.empty(E, dtype=torch.float32, device=d)
    for e in range(E):
        bd = case.b(e, d)
        nv.global_scale(bd, out=gsB[e:e + 1])
        nv.quantize(bd, gsB[e:e + 1], q=Bq[e], sf=sfB[e])
    del bd
    al = nv.alpha(gsA, gsB)
    # a global scale fixed in advance: h of these inputs stays well below 256 in magnitude
    gs_h = np.float32(2688.0 / 256.0)
    off = r.offsets.to(d)
    hq, hsf = _run_gpu(d, Aq, sfA, Bq, sfB, al, off, torch.tensor([gs_h], device=d), rows)
    counts = (r.offsets[1:] - r.offsets[:-1]).numpy()
    rng = np.random.default_rng(case.route_seed)
    nonempty = np.flatnonzero(counts > 0)
    picks = {int(nonempty[np.argmax(counts[nonempty])]), int(nonempty[np.argmin(counts[nonempty])])}
    picks |= set(rng.choice(nonempty, 3, replace=False).tolist())
    blocks = np.array(sorted(set(rng.choice(I // 16, 6, replace=False).tolist()) | {0, I // 16 - 1}))
    j = (blocks[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
    ga = oracle.global_scale(a.numpy())
    for e in sorted(picks):
        r0, r1 = int(r.offsets[e]), int(r.offsets[e + 1])
        b = case.b(e, d).cpu()
        gb = oracle.global_scale(b.numpy())
        qa, sa = oracle.quantize(a[r0:r1].numpy(), ga)
        qg, sg = oracle.quantize(b[j].contiguous().numpy(), gb)
        qu, su = oracle.quantize(b[I + j].contiguous().numpy(), gb)
        alo = oracle.alpha(ga, gb)
        v_g, S_g, _ = oracle.gemm(qa, sa, qg, sg, alo)
        v_u, S_u, _ = oracle.gemm(qa, sa, qu, su, alo)
        _check_sampled(hq[r0:r1], hsf[r0:r1], v_g, v_u, S_g, S_u, alo, gs_h, blocks, K,
                       f"{case.name} expert {e}")


def test_swiglu_rejects_bad_shapes(cuda_device):
    d = cuda_device
    z = torch.zeros(64, dtype=torch.uint8, device=d)
    lib = nv.load()
    args = [z.data_ptr()] * 4 + [z.data_ptr(), z.data_ptr()]
    # I % 64 != 0
    st = lib.nvfp4_grouped_gemm_swiglu(*args, 4, 64, 96, 512, z.data_ptr(), z.data_ptr(), z.data_ptr(), None)
    assert st == 2
    # gs_h missing
    st = lib.nvfp4_grouped_gemm_swiglu(*args, 4, 64, 128, 512, None, z.data_ptr(), z.data_ptr(), None)
    assert st == 1
