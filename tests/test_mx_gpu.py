"""GPU parity of the MXFP4 variant (use_nvfp4=False in the mm_fp4 signature: "The Art of
Reading the Manual", section "The Message") against the CPU oracle (oracle.mx_quantize,
oracle.mx_gemm): OCP MX v1.0 FP4, e2m1 elements with one E8M0 scale per 32 K elements.

* Quantisation: codes and scale bytes bit-exact, both scale layouts, fp32 and bf16 inputs,
  with special blocks (all zero, amax exactly a power of two and just below one, subnormal
  and tiny values, values near the fp32 maximum, mixed signs with values that round to zero).
* Product: within the GEMM tolerance 2^-7 |alpha| sum|a b| + 1e-6 on the configuration shapes
  and ragged ones (few-token tiles, split-K, 128- and 256-wide tiles), and bit-exact where every
  output is one dequantised product (one-hot rows), which also pins which scale byte each of
  the two 64-wide MMAs of a 32-element-block pair reads.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle
from helpers import bf16_bits_of, check_within_tolerance, tile_np

pytestmark = pytest.mark.gpu


def _special_rows(K: int) -> np.ndarray:
    """Rows of blocks that exercise the shared-exponent rule and the code rounding edges."""
    rng = np.random.default_rng(5)
    rows = []
    f32 = np.float32
    blocks = [
        np.zeros(32, f32),                                        # all zero -> byte 0
        np.full(32, 4.0, f32),                                    # amax a power of two
        np.full(32, np.nextafter(f32(4.0), f32(0)), f32),         # just below one
        (rng.standard_normal(32) * 1e-40).astype(f32),            # subnormal inputs
        np.full(32, f32(3.0e38)) * np.sign(rng.standard_normal(32)).astype(f32),   # near max
        np.concatenate([[f32(6.0)], rng.uniform(-0.3, 0.3, 31).astype(f32)]),       # rounds to +-0
        np.concatenate([[f32(7.9)], np.full(31, f32(-7.0))]),     # saturation in (6, 8) * 2^e
        np.array([2.0 ** -127] + [0.0] * 31, f32),                # amax below 2^-126
        np.array([2.0 ** -126] * 32, f32),                        # smallest normal
        np.array([2.0 ** -125] * 32, f32),
        (rng.standard_normal(32) * 2.0 ** 100).astype(f32),
        np.linspace(-6, 6, 32).astype(f32),                       # every code boundary region
    ]
    per_row = K // 32
    for i in range(0, len(blocks), per_row):
        chunk = blocks[i:i + per_row]
        while len(chunk) < per_row:
            chunk.append(rng.standard_normal(32).astype(f32))
        rows.append(np.concatenate(chunk))
    return np.stack(rows)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=str)
@pytest.mark.parametrize("M,K", [(1, 128), (37, 512), (256, 6144), (1024, 2048), (300, 96)])
def test_mx_quantize_bit_exact(cuda_device, dtype, M, K):
    x = workloads.normal(M, K, 1.0, 31 * M + K) * torch.exp2(
        torch.randint(-20, 20, (M, 1), generator=torch.Generator().manual_seed(M)).float())
    if K % 32 == 0 and M >= 2:
        sp = _special_rows(K)
        n = min(len(sp), M)
        x[:n] = torch.from_numpy(sp[:n])
    x = x.to(dtype)
    x32 = x.to(torch.float32).numpy()
    q_o, sf_o = oracle.mx_quantize(x32)
    q, sf = nv.mx_quantize(x.to(cuda_device), tiled=False)
    np.testing.assert_array_equal(sf.cpu().numpy(), sf_o)
    np.testing.assert_array_equal(q.cpu().numpy(), q_o)
    if K % 128 == 0:
        # the tiled layout pads the rows to 128; the quantiser writes only real rows' scales
        sf2 = torch.zeros(nv.mx_sf_bytes(M, K, True), dtype=torch.uint8, device=cuda_device)
        q2, sf2 = nv.mx_quantize(x.to(cuda_device), sf=sf2, tiled=True)
        assert torch.equal(q2, q)
        np.testing.assert_array_equal(sf2.cpu().numpy(), tile_np(sf_o, K // 2))
        np.testing.assert_array_equal(nv.mx_sf_tile(sf).cpu().numpy(), tile_np(sf_o, K // 2))


def _mx_operands(a: torch.Tensor, b: torch.Tensor, dev):
    qa_o, sa_o = oracle.mx_quantize(a.numpy())
    qb_o, sb_o = oracle.mx_quantize(b.numpy())
    qa, sa = nv.mx_quantize(a.to(dev), tiled=True)
    qb, sb = nv.mx_quantize(b.to(dev), tiled=True)
    return (qa, sa, qb, sb), (qa_o, sa_o, qb_o, sb_o)


def _run(dev, a, b, rows=None, cols=None, out_dtype=torch.bfloat16, alpha=1.0):
    M, K = a.shape
    N = b.shape[0]
    (qa, sa, qb, sb), (qa_o, sa_o, qb_o, sb_o) = _mx_operands(a, b, dev)
    al = torch.full((1,), alpha, device=dev)
    big = torch.full((M + 2, N), -12352.0, dtype=out_dtype, device=dev)
    out = nv.mx_gemm(qa, sa, qb, sb, al, out=big[:M], workspace=nv.make_workspace(M, N, K, dev))
    st, code = nv.last_device_error()
    assert st == 0, hex(code)
    assert (big[M:].float() == -12352.0).all(), "write past the last output row"
    if rows is not None:
        qa_o, sa_o = qa_o[rows], sa_o[rows]
        out = out[torch.as_tensor(rows, device=dev)]
    if cols is not None:
        qb_o, sb_o = qb_o[cols], sb_o[cols]
        out = out[:, torch.as_tensor(cols, device=dev)]
    v, S, _ = oracle.mx_gemm(qa_o, sa_o, qb_o, sb_o, alpha)
    check_within_tolerance(out, v, S, alpha, f"mx {M}x{N}x{K}")


@pytest.mark.parametrize("case", [workloads.single_case()] + workloads.attn_proj_cases()
                         + workloads.moe_expert_cases()[::3], ids=lambda c: c.name)
def test_mx_gemm_config_shapes(cuda_device, case):
    rows = None if case.M <= 256 else np.r_[0:48, case.M - 48:case.M]
    _run(cuda_device, case.a(), case.b(), rows=rows)


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (17, 136, 512), (64, 24, 768), (65, 264, 768),
                                   (130, 776, 1024), (300, 512, 4096), (16, 6144, 2048)])
def test_mx_gemm_ragged(cuda_device, M, N, K):
    a = workloads.normal(M, K, 1.0, M * 5 + N)
    b = workloads.normal(N, K, 0.02, N * 3 + K)
    _run(cuda_device, a, b)


def test_mx_gemm_plateau_sampled_and_out_dtypes(cuda_device):
    c = workloads.plateau_cases()[0]
    rng = np.random.default_rng(11)
    rows = np.sort(rng.choice(c.M, 32, replace=False))
    cols = np.sort(rng.choice(c.N, 256, replace=False))
    _run(cuda_device, c.a(), c.b(), rows=rows, cols=cols)
    a = workloads.normal(96, 1024, 1.0, 1)
    b = workloads.normal(264, 1024, 1.0, 2)
    for dt in (torch.float16, torch.float32):
        _run(cuda_device, a, b, out_dtype=dt, alpha=0.5)


@pytest.mark.parametrize("M,N,K", [(16, 768, 6144), (64, 256, 512), (300, 512, 1024), (130, 1024, 2048)])
def test_mx_one_hot_rows_bit_exact(cuda_device, M, N, K):
    rng = np.random.default_rng(M + N)
    ks = rng.integers(0, K, M)
    Aq = np.zeros((M, K // 2), np.uint8)
    for m, k in enumerate(ks):
        Aq[m, k // 2] = 0x2 << (4 * (k % 2))          # code 2 = 1.0
    sfA = np.full((M, K // 32), 127, np.uint8)         # 2^0
    Bq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sfB = rng.integers(115, 140, (N, K // 32), dtype=np.uint8)
    v, S, _ = oracle.mx_gemm(Aq, sfA, Bq, sfB, 1.0)
    want = oracle.bf16_bits(v)
    d = cuda_device
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(d)
    for use_ws in (True, False):
        out = nv.mx_gemm(t(Aq), t(tile_np(sfA, K // 2)), t(Bq), t(tile_np(sfB, K // 2)),
                         torch.ones(1, device=d), workspace=nv.make_workspace(M, N, K, d) if use_ws else None)
        np.testing.assert_array_equal(bf16_bits_of(out), want)
