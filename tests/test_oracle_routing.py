"""Pins for the oracle's MoE routing around the grouped product (top-8 of 256 experts, "When a
Benchmark Crashes", section "Why This Message Was Written"). Each check compares the oracle
with something other than itself:

* route_topk: torch's softmax + topk in fp64 (library), brute-force ordering with the tie
  rule on tied logits, weights that sum to 1.
* permute_by_expert: brute force (Python sorting of (expert, token, slot) triples) on small
  cases, the inverse map, and torch's stable sort as the bench's input generator uses it.
* gather_quantize: equal to quantising every token once and gathering the quantised rows.
* combine: one-hot outputs give back the weights; linearity.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_08_b200 import workloads


def test_route_topk_matches_torch():
    g = torch.Generator().manual_seed(11)
    logits = torch.randn(300, 256, generator=g)
    experts, probs, weights = oracle.route_topk(logits.numpy(), 8)
    p = torch.softmax(logits.double(), dim=-1)
    w, idx = torch.topk(p, 8, dim=-1)
    np.testing.assert_array_equal(experts, idx.numpy())
    np.testing.assert_allclose(probs, w.numpy(), rtol=1e-14)
    np.testing.assert_allclose(weights.sum(axis=1), 1.0, rtol=1e-15)
    assert (np.diff(probs, axis=1) <= 0).all()


def test_route_topk_ties_go_to_the_lower_expert():
    logits = np.zeros((3, 16), np.float32)
    logits[0, [3, 7, 9]] = 2.0                      # three tied leaders
    logits[1, :] = 1.0                              # everything tied
    logits[2, [15, 0]] = [5.0, 5.0]
    experts, _, weights = oracle.route_topk(logits, 4)
    for t in range(3):
        brute = sorted(range(16), key=lambda e: (-float(logits[t, e]), e))[:4]
        assert experts[t].tolist() == brute
    assert experts[0].tolist() == [3, 7, 9, 0] and experts[1].tolist() == [0, 1, 2, 3]
    np.testing.assert_allclose(weights[1], 0.25)


@pytest.mark.parametrize("T,k,E,seed", [(5, 2, 4, 0), (17, 3, 6, 1), (40, 8, 16, 2)])
def test_permute_brute_force(T, k, E, seed):
    experts = np.random.default_rng(seed).integers(0, E, (T, k)).astype(np.int32)
    token, slot, offsets, row_of = oracle.permute_by_expert(experts, E)
    triples = sorted((int(experts[t, s]), t, s) for t in range(T) for s in range(k))
    assert [(int(experts[t, s]), int(t), int(s)) for t, s in zip(token, slot)] == triples
    counts = [sum(1 for e, _, _ in triples if e == x) for x in range(E)]
    assert offsets.tolist() == [0] + list(np.cumsum(counts))
    for t in range(T):
        for s in range(k):
            r = row_of[t, s]
            assert token[r] == t and slot[r] == s
            assert offsets[experts[t, s]] <= r < offsets[experts[t, s] + 1]


def test_permute_matches_the_input_generator():
    # the bench's MoE inputs route with torch.topk and a stable torch.sort; same logits give
    # the same expert-sorted rows and offsets
    route = workloads.routing(512, 4321)
    logits = torch.randn(512, 256, generator=torch.Generator().manual_seed(4321), dtype=torch.float32)
    experts, _, _ = oracle.route_topk(logits.numpy(), 8)
    token, _, offsets, _ = oracle.permute_by_expert(experts, 256)
    np.testing.assert_array_equal(offsets, route.offsets.numpy())
    np.testing.assert_array_equal(token, route.token_of_row.numpy())


def test_gather_quantize_is_quantise_then_gather():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((12, 64)).astype(np.float32)
    experts, _, _ = oracle.route_topk(rng.standard_normal((12, 8)).astype(np.float32), 3)
    token, _, _, _ = oracle.permute_by_expert(experts, 8)
    gs = oracle.global_scale(x)
    q, sf = oracle.gather_quantize(x, token, gs)
    q_all, sf_all = oracle.quantize(x, gs)
    np.testing.assert_array_equal(q, q_all[token])
    np.testing.assert_array_equal(sf, sf_all[token])


def test_combine_one_hot_and_linearity():
    rng = np.random.default_rng(6)
    T, k, E = 10, 3, 5
    experts, _, weights = oracle.route_topk(rng.standard_normal((T, E)).astype(np.float32), k)
    token, slot, _, row_of = oracle.permute_by_expert(experts, E)
    # y[r] = one-hot of (token, slot) over T * k columns: out[t] holds t's weights
    y = np.zeros((T * k, T * k))
    y[np.arange(T * k), token * k + slot] = 1.0
    out = oracle.combine(y, weights, row_of)
    for t in range(T):
        np.testing.assert_array_equal(out[t].reshape(T, k)[t], weights[t])
        assert out[t].sum() == pytest.approx(1.0, rel=1e-15)
    y1, y2 = rng.standard_normal((T * k, 4)), rng.standard_normal((T * k, 4))
    np.testing.assert_allclose(oracle.combine(y1 + 2 * y2, weights, row_of),
                               oracle.combine(y1, weights, row_of) + 2 * oracle.combine(y2, weights, row_of),
                               rtol=1e-13, atol=1e-13)
