"""Write tests/golden/oracle_next_regression.json from the CPU oracle alone.

Freezes the oracle's results for the steps that the CUDA library does not implement yet
(MXFP4, the fp16 output rounding, SwiGLU + requantise, MoE routing) on seeded inputs, so
that a later change to their arithmetic fails a test and has to be made deliberately. Like
oracle_regression.json it does not pin the oracle to the reference pages, which print no
reproducible example; the pins are the tests in tests/test_oracle*.py.

Run: python tests/golden/make_oracle_next_regression.py
"""
import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from nvfp4_block_scaled_08_b200 import workloads  # noqa: E402


def _h(arr) -> str:
    return hashlib.sha256(np.ascontiguousarray(arr).tobytes()).hexdigest()


def compute():
    case = workloads.single_case()                     # 128 x 256 x 512, N(0,1)
    a = case.a().numpy()
    b = case.b().numpy()
    # MXFP4 operands and product
    qa, sa = oracle.mx_quantize(a)
    qb, sb = oracle.mx_quantize(b)
    v_mx, S_mx, exact_mx = oracle.mx_gemm(qa, sa, qb, sb, 1.0)
    # NVFP4 product, rounded to fp16 instead of bf16
    ga, gb = oracle.global_scale(a), oracle.global_scale(b)
    Aq, sfA = oracle.quantize(a, ga)
    Bq, sfB = oracle.quantize(b, gb)
    v, _, _ = oracle.gemm(Aq, sfA, Bq, sfB, oracle.alpha(ga, gb))
    # SwiGLU + requantise of that product read as a gate_up output (I = 128)
    q_h, sf_h, h = oracle.swiglu_quantize(v, np.float32(64.0))
    # routing of 64 tokens over 16 experts, top 4
    logits = workloads.normal(64, 16, 1.0, 2468).numpy()
    experts, _, weights = oracle.route_topk(logits, 4)
    token, slot, offsets, row_of = oracle.permute_by_expert(experts, 16)
    return {
        "case": case.name,
        "mx": {"sha256_qa": _h(qa), "sha256_sa": _h(sa), "sha256_qb": _h(qb), "sha256_sb": _h(sb),
               "sha256_v": _h(v_mx), "exact": bool(exact_mx),
               "v_0_0": float(v_mx[0, 0]), "S_5_17": float(S_mx[5, 17])},
        "fp16": {"sha256_out_fp16_bits": _h(oracle.fp16_bits(v))},
        "swiglu": {"sha256_q": _h(q_h), "sha256_sf": _h(sf_h), "h_samples": [float(h[0, 0]), float(h[77, 101])]},
        # weights go through exp: sampled and compared with a tolerance, not hashed
        "routing": {"sha256_experts": _h(experts),
                    "weights_samples": [float(weights[t, s]) for t, s in ((0, 0), (10, 2), (63, 3))],
                    "offsets": offsets.tolist(), "sha256_token": _h(token), "sha256_slot": _h(slot),
                    "sha256_row_of": _h(row_of)},
    }


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_next_regression.json")
    with open(out, "w") as f:
        json.dump(compute(), f, indent=1)
    print("wrote", out)
