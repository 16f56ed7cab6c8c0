"""The backward and masked oracles still reproduce their committed small
fixtures (tests/golden/, written by tests/golden/gen_golden.py from the
oracles only): regression checks next to the pins, which are what tie the
oracles to the definition."""
import json
import os

import numpy as np

import oracle

HERE = os.path.join(os.path.dirname(__file__), "golden")
NAMES = ("q", "k", "v", "tq", "tk", "tv")
GRADS = ("dq", "dk", "dv", "dtq", "dtk", "dtv")


def _inputs():
    g = json.load(open(os.path.join(HERE, "oracle_small.json")))
    return [np.array(g[n], dtype=np.float64) for n in NAMES], g["scale"]


def _close(a, b):
    return np.allclose(np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64), rtol=0, atol=1e-14)


def test_backward_golden():
    arrs, s = _inputs()
    g = json.load(open(os.path.join(HERE, "oracle_bwd_small.json")))
    got = oracle.attn_jvp_bwd(*arrs, np.array(g["dout"]), np.array(g["dtout"]), s)
    for n in GRADS:
        assert _close(got[n], g[n]), n


def test_masked_golden():
    arrs, s = _inputs()
    gb = json.load(open(os.path.join(HERE, "oracle_bwd_small.json")))
    do, dto = np.array(gb["dout"]), np.array(gb["dtout"])
    g = json.load(open(os.path.join(HERE, "oracle_masked_small.json")))
    co, cto, clse = oracle.attn_jvp_causal(*arrs, s)
    cg = oracle.attn_jvp_bwd_causal(*arrs, do, dto, s)
    for got, key in ((co, "o"), (cto, "to"), (clse, "lse")):
        assert _close(got, g["causal"][key]), key
    for n in GRADS:
        assert _close(cg[n], g["causal"][n]), n
    po, pto, plse = oracle.attn_jvp_packed(*arrs, s, g["cu_q"], g["cu_k"], False)
    pg = oracle.attn_jvp_bwd_packed(*arrs, do, dto, s, g["cu_q"], g["cu_k"], False)
    for got, key in ((po, "o"), (pto, "to"), (plse, "lse")):
        assert _close(got, g["packed"][key]), key
    for n in GRADS:
        assert _close(pg[n], g["packed"][n]), n
