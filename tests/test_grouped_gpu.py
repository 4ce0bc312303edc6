"""GPU parity of the grouped (mixture-of-experts) NVFP4 GEMM against the CPU oracle.

Small cases run the oracle over every expert (including empty experts and ragged row
counts). The four full-size configs (256 experts, top-8 routing of 512 or 4096 tokens,
gate_up 4096 x 6144 and down 6144 x 2048) run in the benchmark's launch configuration and
are checked on sampled experts and sampled output columns."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle
from helpers import check_within_tolerance

pytestmark = pytest.mark.gpu


def _small_case(dev, counts, N, K, seed, pad_rows=0):
    E = len(counts)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(off[-1]) + pad_rows
    a = workloads.normal(max(rows, 1), K, 1.0, seed)[:rows]
    bs = [workloads.normal(N, K, 0.02, seed + 100 + e) for e in range(E)]
    # CUDA path
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
    sentinel = 776.0   # exactly representable in bf16
    out = torch.full((rows, N), sentinel, dtype=torch.bfloat16, device=dev)
    nv.grouped_gemm(Aq, sfA, Bq, sfB, al, torch.from_numpy(off).to(dev), out=out)
    st, code = nv.last_device_error()
    assert st == 0, hex(code)
    # oracle
    ga = oracle.global_scale(a.numpy())
    qa, sa = oracle.quantize(a.numpy(), ga)
    qb = np.stack([oracle.quantize(b.numpy(), oracle.global_scale(b.numpy()))[0] for b in bs])
    sb = np.stack([oracle.quantize(b.numpy(), oracle.global_scale(b.numpy()))[1] for b in bs])
    alo = np.array([oracle.alpha(ga, oracle.global_scale(b.numpy())) for b in bs], np.float32)
    np.testing.assert_array_equal(al.cpu().numpy(), alo)
    v, S, _ = oracle.grouped_gemm(qa, sa, qb, sb, alo, off)
    used = int(off[-1])
    for e in range(E):
        r0, r1 = off[e], off[e + 1]
        if r1 > r0:
            check_within_tolerance(out[r0:r1], v[r0:r1], S[r0:r1], alo[e], f"expert {e}")
    # rows past the last expert are never written
    if pad_rows:
        assert (out[used:].float() == sentinel).all()


def test_grouped_small_ragged_and_empty(cuda_device):
    _small_case(cuda_device, [3, 0, 17, 1, 40, 0, 0, 129, 16, 33], 256, 512, 11, pad_rows=5)


def test_grouped_single_expert_and_all_empty_but_one(cuda_device):
    _small_case(cuda_device, [0, 0, 70, 0], 136, 256, 12)
    _small_case(cuda_device, [300], 128, 768, 13)


@pytest.mark.parametrize("rows_each", [16, 128, 160, 200])
def test_grouped_token_tile_widths(cuda_device, rows_each):
    # mean rows per expert drives the token-tile width (32, 64, 128, 176 or 256); at 160 the
    # 176-row tiles (two 88-row boxes) hold 157..165 rows
    _small_case(cuda_device, [rows_each - 3, rows_each, rows_each + 5, rows_each - 1], 384, 1024,
                rows_each)


@pytest.mark.parametrize("grouped_bn", [32, 64, 128, 176, 256])
def test_grouped_every_forced_tile_width(cuda_device, grouped_bn):
    # ragged experts (empty, 1 row, a tile and a bit, several tiles) in every token-tile width
    with nv.plan_override(grouped_bn=grouped_bn):
        _small_case(cuda_device, [0, 1, 177, 90, 3, 400, 0, 33], 264, 512, 40 + grouped_bn, pad_rows=3)


def _full_config(dev, case: workloads.GroupedCase, n_experts_checked=5, n_cols=192):
    r = case.route()
    rows = r.rows
    a = case.a(rows)
    ad = a.to(dev)
    gsA = nv.global_scale(ad)
    Aq, sfA = nv.quantize(ad, gsA)
    del ad
    E, N, K = case.num_experts, case.N, case.K
    Bq = torch.empty(E, N, K // 2, dtype=torch.uint8, device=dev)
    sfB = torch.empty(E, N, K // 16, dtype=torch.uint8, device=dev)
    gsB = torch.empty(E, dtype=torch.float32, device=dev)
    for e in range(E):
        bd = case.b(e, dev)
        nv.global_scale(bd, out=gsB[e:e + 1])
        nv.quantize(bd, gsB[e:e + 1], q=Bq[e], sf=sfB[e])
    del bd
    al = nv.alpha(gsA, gsB)
    off = r.offsets.to(dev)
    out = nv.grouped_gemm(Aq, sfA, Bq, sfB, al, off)
    st, code = nv.last_device_error()
    assert st == 0, hex(code)
    # oracle on sampled experts x sampled weight rows (output columns)
    counts = (r.offsets[1:] - r.offsets[:-1]).numpy()
    rng = np.random.default_rng(case.route_seed)
    nonempty = np.flatnonzero(counts > 0)
    picks = {int(nonempty[np.argmax(counts[nonempty])]), int(nonempty[np.argmin(counts[nonempty])]),
             0, E - 1}
    picks |= set(rng.choice(nonempty, n_experts_checked, replace=False).tolist())
    ga = oracle.global_scale(a.numpy())
    cols = np.array(sorted(set(rng.choice(N, n_cols - 2, replace=False).tolist()) | {0, N - 1}))
    for e in sorted(picks):
        r0, r1 = int(r.offsets[e]), int(r.offsets[e + 1])
        if r1 == r0:
            continue
        b = case.b(e, dev).cpu()            # the seeded generator's fp32 weights
        gb = oracle.global_scale(b.numpy())
        assert np.float32(gsB[e].item()) == gb
        qa, sa = oracle.quantize(a[r0:r1].numpy(), ga)
        qb, sb = oracle.quantize(b[cols].contiguous().numpy(), gb)
        alo = oracle.alpha(ga, gb)
        v, S, _ = oracle.gemm(qa, sa, qb, sb, alo)
        got = out[r0:r1][:, torch.as_tensor(cols, device=dev)]
        check_within_tolerance(got, v, S, alo, f"{case.name} expert {e}")


@pytest.mark.parametrize("case", workloads.grouped_cases(), ids=lambda c: c.name)
def test_grouped_full_configs_sampled(cuda_device, case):
    _full_config(cuda_device, case)
