"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and arranges them into the shapes of the reference
pages' workloads. It holds none of the method's arithmetic (no scaling, rounding,
packing or products), so both the CUDA path and the CPU oracle can consume it.

Shapes (GLM-5-NVFP4 layer shapes: hidden 6144, MoE intermediate 2048, 256 experts,
top-8; "When a Benchmark Crashes", sections "Why This Message Was Written" and "Input
Knowledge Required", item 1; the benchmark grid M in {16..1024}, N in {768, 2048},
K = 6144 from section "Assumptions Made", item 3):

* ``single``      : M=128, N=256, K=512, A and B ~ N(0, 1).
* ``attn_proj``   : N=768, K=6144, M in {16, 64, 256, 1024}; A ~ N(0,1), B ~ N(0,0.02).
* ``moe_expert``  : up N=2048 K=6144 and down N=6144 K=2048, M in {16,...,1024}.
* ``moe_grouped`` : 256 experts, top-8 routing of T in {512, 4096} tokens from a softmax
                    over N(0,1) router logits; gate_up N=4096 K=6144, down N=6144 K=2048.
* ``plateau``     : M=N=K in {4096, 8192, 16384}, U(-1, 1); plus 512 x 2048 x 6144.

All draws use a CPU ``torch.Generator`` seeded with ``1234 + config index`` (plus a
per-tensor offset), so every run and every process sees identical inputs.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

SEED_BASE = 1234
HIDDEN = 6144
MOE_INTER = 2048
NUM_EXPERTS = 256
TOP_K = 8


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(rows: int, cols: int, std: float, seed: int) -> torch.Tensor:
    """fp32 [rows, cols] ~ N(0, std^2), drawn on the CPU."""
    return torch.randn(rows, cols, generator=_gen(seed), dtype=torch.float32) * std


def uniform(rows: int, cols: int, seed: int) -> torch.Tensor:
    """fp32 [rows, cols] ~ U(-1, 1), drawn on the CPU."""
    return torch.rand(rows, cols, generator=_gen(seed), dtype=torch.float32) * 2.0 - 1.0


@dataclass
class GemmCase:
    name: str
    M: int
    N: int
    K: int
    a_std: float | None   # None: uniform(-1, 1)
    b_std: float | None
    seed: int

    def a(self) -> torch.Tensor:
        if self.a_std is None:
            return uniform(self.M, self.K, self.seed)
        return normal(self.M, self.K, self.a_std, self.seed)

    def b(self) -> torch.Tensor:
        if self.b_std is None:
            return uniform(self.N, self.K, self.seed + 1)
        return normal(self.N, self.K, self.b_std, self.seed + 1)

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K


def single_case() -> GemmCase:
    return GemmCase("single_128x256x512", 128, 256, 512, 1.0, 1.0, SEED_BASE + 0)


def attn_proj_cases() -> list[GemmCase]:
    return [GemmCase(f"attn_proj_M{m}", m, 768, HIDDEN, 1.0, 0.02, SEED_BASE + 1 + 10 * i)
            for i, m in enumerate((16, 64, 256, 1024))]


def moe_expert_cases() -> list[GemmCase]:
    out = []
    for i, m in enumerate((16, 32, 64, 128, 512, 1024)):
        out.append(GemmCase(f"moe_up_M{m}", m, MOE_INTER, HIDDEN, 1.0, 0.02,
                            SEED_BASE + 2 + 10 * i))
        out.append(GemmCase(f"moe_down_M{m}", m, HIDDEN, MOE_INTER, 1.0, 0.02,
                            SEED_BASE + 2 + 10 * i + 5))
    return out


def plateau_cases() -> list[GemmCase]:
    out = [GemmCase(f"square_{s}", s, s, s, None, None, SEED_BASE + 4 + 10 * i)
           for i, s in enumerate((4096, 8192, 16384))]
    out.append(GemmCase("ratio_512x2048x6144", 512, 2048, 6144, None, None, SEED_BASE + 44))
    return out


@dataclass
class Routing:
    """Token-to-expert assignment sorted by expert (counting-sort order).

    ``token_of_row[r]`` is the token that row r of the expert-sorted activation matrix
    comes from; ``offsets[e]:offsets[e+1]`` are expert e's rows; ``weights[r]`` is the
    router probability of that (token, expert) pair.
    """
    T: int
    offsets: torch.Tensor        # int32 [E + 1]
    token_of_row: torch.Tensor   # int64 [T * top_k]
    weights: torch.Tensor        # fp32 [T * top_k]

    @property
    def rows(self) -> int:
        return int(self.offsets[-1])


def routing(T: int, seed: int, num_experts: int = NUM_EXPERTS, top_k: int = TOP_K) -> Routing:
    """Top-k routing from a softmax over N(0,1) logits, then a stable sort by expert."""
    logits = torch.randn(T, num_experts, generator=_gen(seed), dtype=torch.float32)
    probs = torch.softmax(logits, dim=-1)
    w, idx = torch.topk(probs, top_k, dim=-1)                   # [T, top_k]
    expert = idx.reshape(-1)
    token = torch.arange(T).repeat_interleave(top_k)
    order = torch.sort(expert, stable=True).indices
    counts = torch.bincount(expert, minlength=num_experts)
    offsets = torch.zeros(num_experts + 1, dtype=torch.int32)
    offsets[1:] = torch.cumsum(counts, 0).to(torch.int32)
    return Routing(T, offsets, token[order], w.reshape(-1)[order])


@dataclass
class GroupedCase:
    """One grouped-GEMM workload. Routing and activations are drawn on the CPU; the
    expert weights (up to 25 GB of fp32 for 256 experts) are drawn per expert by torch's
    seeded generator on the device that will quantise them. Weight seeds depend only on the
    projection, so both token counts see the same model weights."""
    name: str
    T: int
    N: int
    K: int
    route_seed: int
    weight_seed: int
    num_experts: int = NUM_EXPERTS

    def route(self) -> Routing:
        return routing(self.T, self.route_seed, self.num_experts)

    def a(self, rows: int) -> torch.Tensor:
        """Expert-sorted activations [rows, K] ~ N(0, 1) (CPU)."""
        return normal(rows, self.K, 1.0, self.route_seed + 1)

    def b(self, expert: int, device="cpu") -> torch.Tensor:
        """Expert weights [N, K] ~ N(0, 0.02^2), drawn on `device`."""
        g = torch.Generator(device=device)
        g.manual_seed(self.weight_seed * 4096 + expert)
        return torch.randn(self.N, self.K, generator=g, dtype=torch.float32, device=device) * 0.02

    @property
    def flops_per_row(self) -> int:
        return 2 * self.N * self.K


def grouped_cases() -> list[GroupedCase]:
    out = []
    for i, T in enumerate((512, 4096)):
        out.append(GroupedCase(f"moe_gate_up_T{T}", T, 2 * MOE_INTER, HIDDEN,
                               SEED_BASE + 3 + 10 * i, SEED_BASE + 3))
        out.append(GroupedCase(f"moe_down_T{T}", T, HIDDEN, MOE_INTER,
                               SEED_BASE + 3 + 10 * i + 5, SEED_BASE + 8))
    return out
