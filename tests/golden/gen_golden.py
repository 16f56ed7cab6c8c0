"""Writes tests/golden/oracle_small.json: a small attention-JVP case whose
expected values come from the fp64 oracle only (a regression fixture; the
pages print no worked example).  Inputs are small dyadic rationals written out
here, so they are exact in fp32, bf16 and fp64.

Run from the repository root:  python tests/golden/gen_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402

Q = [[[0.5, -1.0], [1.25, 0.25], [-0.75, 2.0]]]
K = [[[1.0, 0.5], [-0.5, 1.5], [0.25, -1.0], [2.0, 0.0]]]
V = [[[0.5, 1.0], [-1.0, 0.25], [1.5, -0.5], [0.0, 2.0]]]
TQ = [[[0.25, 0.5], [-0.5, 0.0], [1.0, -0.25]]]
TK = [[[0.0, -0.5], [0.75, 0.25], [-1.0, 0.5], [0.5, 1.0]]]
TV = [[[1.0, 0.0], [0.5, -0.5], [-0.25, 1.0], [0.75, 0.25]]]
SCALE = 0.5

if __name__ == "__main__":
    arrs = [np.array(x, dtype=np.float64) for x in (Q, K, V, TQ, TK, TV)]
    o, to, lse = oracle.attn_jvp(*arrs, SCALE)
    out = {"about": "fp64 oracle output for the inputs below (regression fixture)",
           "scale": SCALE, "q": Q, "k": K, "v": V, "tq": TQ, "tk": TK, "tv": TV,
           "o": o.tolist(), "to": to.tolist(), "lse": lse.tolist()}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)
