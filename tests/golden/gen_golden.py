"""Writes the small regression fixtures of tests/golden/, whose expected
values come from the fp64 oracles only (the pages print no worked example):
oracle_small.json (attention + JVP), oracle_bwd_small.json (its backward for
the cotangents below) and oracle_masked_small.json (the causal forward and
backward on the same inputs, bottom-right aligned, and a packed pair of
sequences).  Inputs are small dyadic rationals written out here, so they are
exact in fp32, bf16 and fp64.

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
DO = [[[1.0, -0.5], [0.25, 0.75], [-1.25, 0.5]]]
DTO = [[[-0.5, 0.25], [1.0, 0.0], [0.5, -1.0]]]
# packed: sequence 0 = query rows 0-1 with keys 0-2, sequence 1 = query row 2 with key 3
CU_Q, CU_K = [0, 2, 3], [0, 3, 4]

if __name__ == "__main__":
    arrs = [np.array(x, dtype=np.float64) for x in (Q, K, V, TQ, TK, TV)]
    o, to, lse = oracle.attn_jvp(*arrs, SCALE)
    out = {"about": "fp64 oracle output for the inputs below (regression fixture)",
           "scale": SCALE, "q": Q, "k": K, "v": V, "tq": TQ, "tk": TK, "tv": TV,
           "o": o.tolist(), "to": to.tolist(), "lse": lse.tolist()}
    here = os.path.dirname(os.path.abspath(__file__))
    path = os.path.join(here, "oracle_small.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)
    do, dto = (np.array(x, dtype=np.float64) for x in (DO, DTO))
    g = oracle.attn_jvp_bwd(*arrs, do, dto, SCALE)
    out = {"about": "fp64 backward oracle: gradients of <dout, O> + <dtout, tO> (regression fixture)",
           "scale": SCALE, "dout": DO, "dtout": DTO, **{n: g[n].tolist() for n in g}}
    path = os.path.join(here, "oracle_bwd_small.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)
    co, cto, clse = oracle.attn_jvp_causal(*arrs, SCALE)
    cg = oracle.attn_jvp_bwd_causal(*arrs, do, dto, SCALE)
    po, pto, plse = oracle.attn_jvp_packed(*arrs, SCALE, CU_Q, CU_K, False)
    pg = oracle.attn_jvp_bwd_packed(*arrs, do, dto, SCALE, CU_Q, CU_K, False)
    out = {"about": "fp64 masked oracles: causal (bottom-right aligned) and packed forward and backward "
                    "(regression fixture)",
           "scale": SCALE, "cu_q": CU_Q, "cu_k": CU_K,
           "causal": {"o": co.tolist(), "to": cto.tolist(), "lse": clse.tolist(), **{n: cg[n].tolist() for n in cg}},
           "packed": {"o": po.tolist(), "to": pto.tolist(), "lse": plse.tolist(), **{n: pg[n].tolist() for n in pg}}}
    path = os.path.join(here, "oracle_masked_small.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)
