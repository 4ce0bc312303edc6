"""Write tests/golden/oracle_regression.json from the CPU oracle alone.

The reference pages print no reproducible worked example (their one printed GEMM output
used unseeded random scale bytes), so this fixture does not pin the oracle to the pages;
it freezes the oracle's own results on the 128 x 256 x 512 case so that any later change
to its arithmetic shows up as a test failure and has to be made deliberately.

Run: python tests/golden/make_oracle_regression.py
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


def compute():
    case = workloads.single_case()
    a = case.a().numpy()
    b = case.b().numpy()
    ga, gb = oracle.global_scale(a), oracle.global_scale(b)
    Aq, sfA = oracle.quantize(a, ga)
    Bq, sfB = oracle.quantize(b, gb)
    al = oracle.alpha(ga, gb)
    v, S, exact = oracle.gemm(Aq, sfA, Bq, sfB, al)
    bits = oracle.bf16_bits(v)
    h = lambda arr: hashlib.sha256(np.ascontiguousarray(arr).tobytes()).hexdigest()
    picks = [(0, 0), (5, 17), (127, 255), (64, 128), (100, 3)]
    return {
        "case": case.name,
        "gs_a": float(ga), "gs_b": float(gb), "alpha": float(al),
        "sha256_Aq": h(Aq), "sha256_sfA": h(sfA), "sha256_Bq": h(Bq), "sha256_sfB": h(sfB),
        "sha256_out_bf16_bits": h(bits),
        "exact": bool(exact),
        "samples": [{"m": m, "n": n, "v": float(v[m, n]), "S": float(S[m, n])} for m, n in picks],
    }


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_regression.json")
    with open(out, "w") as f:
        json.dump(compute(), f, indent=1)
    print("wrote", out)
