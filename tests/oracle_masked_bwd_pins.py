"""Checks that pin the fp64 masked / packed backward oracle to facts other
than itself.

Each pin takes a backward callable
``g(q, k, v, tq, tk, tv, dout, dtout, scale, cu_q, cu_k, causal, qrows=None,
krows=None) -> dict`` over packed [H, T, d] tensors (dq, dk, dv, dtq, dtk, dtv
as fp64 arrays) and returns (ok, detail).  The gradients are those of
L = <dout, O> + <dtout, tO>, O and tO being the masked attention and its JVP
(key j of a sequence visible to its query row i iff j <= i + (Lk - Lq) when
causal; rows with no visible key give O = tO = 0).  A plausible slip in the
oracle (the mask off by one, the offset's sign, keys of the wrong sequence,
a dropped chain-rule term) fails at least one pin;
tests/test_oracle_masked_bwd.py plants such slips and checks that.

What pins what:
  finite_difference     <grad, e> equals the central difference of L (the
                        masked forward oracle, itself pinned) along a random
                        e, for each of the six inputs: causal with Lq = Lk,
                        Lq < Lk and Lq > Lk (rows with no key), packed
                        sequences with and without the causal mask.
  torch_reverse_jvp     all six gradients equal torch.autograd through
                        torch.func.jvp of a softmax attention whose hidden
                        scores are -inf (fp64), dense causal and packed.
  unmasked_sequence     one unmasked sequence equals the unmasked backward
                        oracle (itself pinned).
  last_row_sees_all     the last query row of a causal problem sees every
                        key: its dq, dtq equal those of that row alone,
                        unmasked (the unmasked backward oracle).
  sequence_independence a packed batch equals each sequence run alone.
  empty_rows            rows with no visible key get dq = dtq = 0 and their
                        cotangents change no gradient.
  subsets               listed rows / keys equal the rows of the full result.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

NAMES = ("dq", "dk", "dv", "dtq", "dtk", "dtv")
INPUTS = ("q", "k", "v", "tq", "tk", "tv")


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = max(float(np.max(np.abs(b))), 1e-300)
    return float(np.max(np.abs(a - b))) / den


def _inputs(rng, H, Tq, Tk, d):
    return {n: rng.standard_normal((H, Tq if n in ("q", "tq", "dout", "dtout") else Tk, d))
            for n in ("q", "k", "v", "tq", "tk", "tv", "dout", "dtout")}


def _call(g, x, s, cu_q, cu_k, causal, **kw):
    return g(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], x["dout"], x["dtout"], s, cu_q, cu_k, causal, **kw)


def _loss(x, s, cu_q, cu_k, causal):
    o, to, _ = oracle.attn_jvp_packed(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], s, cu_q, cu_k, causal)
    return float(np.sum(o * x["dout"]) + np.sum(to * x["dtout"]))


# (H, d, cu_q, cu_k, causal): one dense causal sequence (square, fewer
# queries, more queries -- the first rows then see no key) and packed batches
CASES = (
    (2, 4, [0, 6], [0, 6], True),
    (1, 5, [0, 4], [0, 9], True),
    (1, 3, [0, 8], [0, 5], True),
    (2, 4, [0, 3, 3, 8], [0, 4, 6, 9], False),
    (1, 4, [0, 5, 7, 12], [0, 3, 8, 10], True),
)


def finite_difference(g):
    rng = np.random.default_rng(21)
    worst = 0.0
    for H, d, cu_q, cu_k, causal in CASES:
        x = _inputs(rng, H, cu_q[-1], cu_k[-1], d)
        s = 0.6
        grads = _call(g, x, s, cu_q, cu_k, causal)
        eps = 1e-6
        for name, gname in zip(INPUTS, NAMES):
            e = rng.standard_normal(x[name].shape)
            xp, xm = dict(x), dict(x)
            xp[name] = x[name] + eps * e
            xm[name] = x[name] - eps * e
            fd = (_loss(xp, s, cu_q, cu_k, causal) - _loss(xm, s, cu_q, cu_k, causal)) / (2 * eps)
            an = float(np.sum(grads[gname] * e))
            scale = float(np.linalg.norm(grads[gname]) * np.linalg.norm(e)) + 1e-30
            worst = max(worst, abs(fd - an) / scale)
    return worst < 1e-7, f"worst |fd - <g,e>| / (|g||e|) = {worst:.2e}"


def _visible(cu_q, cu_k, causal):
    """[Tq, Tk] boolean: packed key column visible to packed query row."""
    Tq, Tk = cu_q[-1], cu_k[-1]
    m = np.zeros((Tq, Tk), dtype=bool)
    for b in range(len(cu_q) - 1):
        lq, lk = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        for i in range(lq):
            nv = lk if not causal else max(0, min(lk, i + (lk - lq) + 1))
            m[cu_q[b] + i, cu_k[b]:cu_k[b] + nv] = True
    return m


def _torch_grads(x, s, cu_q, cu_k, causal):
    vis = torch.tensor(_visible(cu_q, cu_k, causal))
    t = {n: torch.tensor(x[n], dtype=torch.float64, requires_grad=n in INPUTS) for n in x}

    def attn(q, k, v):
        sc = (s * q @ k.mT).masked_fill(~vis, float("-inf"))
        return torch.softmax(sc, dim=-1) @ v

    o, to = torch.func.jvp(attn, (t["q"], t["k"], t["v"]), (t["tq"], t["tk"], t["tv"]))
    loss = (o * t["dout"]).sum() + (to * t["dtout"]).sum()
    gr = torch.autograd.grad(loss, [t[n] for n in INPUTS])
    return dict(zip(NAMES, (a.numpy() for a in gr)))


def torch_reverse_jvp(g):
    rng = np.random.default_rng(22)
    worst = 0.0
    # every query row sees at least one key (the library softmax of an all -inf
    # row is not defined)
    for H, d, cu_q, cu_k, causal in ((2, 5, [0, 7], [0, 7], True), (1, 3, [0, 5], [0, 9], True),
                                     (2, 4, [0, 4, 9], [0, 6, 8], False), (1, 4, [0, 3, 8], [0, 5, 11], True)):
        x = _inputs(rng, H, cu_q[-1], cu_k[-1], d)
        got = _call(g, x, 0.45, cu_q, cu_k, causal)
        ref = _torch_grads(x, 0.45, cu_q, cu_k, causal)
        worst = max(worst, max(_rel(got[n], ref[n]) for n in NAMES))
    return worst < 1e-10, f"worst rel err {worst:.2e}"


def unmasked_sequence(g):
    rng = np.random.default_rng(23)
    x = _inputs(rng, 2, 6, 9, 4)
    got = _call(g, x, 0.7, [0, 6], [0, 9], False)
    ref = oracle.attn_jvp_bwd(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], x["dout"], x["dtout"], 0.7)
    err = max(_rel(got[n], ref[n]) for n in NAMES)
    return err < 1e-12, f"rel err {err:.2e}"


def last_row_sees_all(g):
    rng = np.random.default_rng(24)
    worst = 0.0
    for Lq, Lk in ((6, 6), (4, 9), (8, 5)):
        x = _inputs(rng, 2, Lq, Lk, 4)
        got = _call(g, x, 0.5, [0, Lq], [0, Lk], True)
        last = {n: (x[n][:, -1:] if n in ("q", "tq", "dout", "dtout") else x[n]) for n in x}
        ref = oracle.attn_jvp_bwd(last["q"], last["k"], last["v"], last["tq"], last["tk"], last["tv"],
                                  last["dout"], last["dtout"], 0.5)
        worst = max(worst, _rel(got["dq"][:, -1:], ref["dq"]), _rel(got["dtq"][:, -1:], ref["dtq"]))
    return worst < 1e-12, f"rel err {worst:.2e}"


def sequence_independence(g):
    rng = np.random.default_rng(25)
    worst = 0.0
    for causal in (False, True):
        cu_q, cu_k = [0, 4, 4, 9, 12], [0, 5, 7, 10, 16]
        x = _inputs(rng, 2, cu_q[-1], cu_k[-1], 3)
        full = _call(g, x, 0.55, cu_q, cu_k, causal)
        for b in range(len(cu_q) - 1):
            qs, ks = slice(cu_q[b], cu_q[b + 1]), slice(cu_k[b], cu_k[b + 1])
            lq, lk = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
            if lk == 0:
                continue
            y = {n: (x[n][:, qs] if n in ("q", "tq", "dout", "dtout") else x[n][:, ks]) for n in x}
            one = _call(g, y, 0.55, [0, lq], [0, lk], causal)
            for n in ("dq", "dtq"):
                if lq:
                    worst = max(worst, _rel(full[n][:, qs], one[n]) if np.any(one[n]) else
                                float(np.max(np.abs(full[n][:, qs]))))
            for n in ("dk", "dv", "dtk", "dtv"):
                worst = max(worst, _rel(full[n][:, ks], one[n]) if np.any(one[n]) else
                            float(np.max(np.abs(full[n][:, ks]))))
    return worst < 1e-12, f"worst rel err {worst:.2e}"


def empty_rows(g):
    rng = np.random.default_rng(26)
    Lq, Lk = 9, 4  # causal: rows 0 .. 4 see no key
    x = _inputs(rng, 2, Lq, Lk, 4)
    a = _call(g, x, 0.6, [0, Lq], [0, Lk], True)
    zero = all(np.all(a[n][:, :Lq - Lk] == 0.0) for n in ("dq", "dtq"))
    y = dict(x)
    for n in ("dout", "dtout"):
        y[n] = x[n].copy()
        y[n][:, :Lq - Lk] = rng.standard_normal(y[n][:, :Lq - Lk].shape) * 5.0
    b = _call(g, y, 0.6, [0, Lq], [0, Lk], True)
    same = all(np.array_equal(a[n], b[n]) for n in NAMES)
    nonzero = all(np.any(a[n][:, Lq - Lk:] != 0.0) for n in ("dq", "dtq"))
    return zero and same and nonzero, f"empty-row grads zero: {zero}, cotangents ignored: {same}, others: {nonzero}"


def subsets(g):
    rng = np.random.default_rng(27)
    cu_q, cu_k = [0, 5, 11], [0, 7, 10]
    x = _inputs(rng, 2, cu_q[-1], cu_k[-1], 4)
    full = _call(g, x, 0.5, cu_q, cu_k, True)
    qr, kr = [10, 0, 6], [9, 2, 7]
    sub = _call(g, x, 0.5, cu_q, cu_k, True, qrows=qr, krows=kr)
    ok = all(np.array_equal(sub[n], full[n][:, qr]) for n in ("dq", "dtq"))
    ok = ok and all(np.array_equal(sub[n], full[n][:, kr]) for n in ("dk", "dv", "dtk", "dtv"))
    return ok, "subset rows equal the full result's rows" if ok else "subset mismatch"


ALL_PINS = {f.__name__: f for f in (finite_difference, torch_reverse_jvp, unmasked_sequence, last_row_sees_all,
                                     sequence_independence, empty_rows, subsets)}


def run_all(g):
    out = {}
    for name, fn in ALL_PINS.items():
        try:
            out[name] = fn(g)
        except Exception as e:  # a broken oracle may also fail by raising
            out[name] = (False, f"raised {type(e).__name__}: {e}")
    return out
