"""Checks that pin the masked / packed fp64 oracle (oracle.attn_jvp_packed) to
facts other than itself.

Each pin takes a callable ``f(q, k, v, tq, tk, tv, scale, cu_q, cu_k, causal)``
on packed [H, T, d] arrays and returns (ok, detail):
  prefix_property       causal row i equals the unmasked oracle (pinned on its
                        own) on keys 0 .. i + Lk - Lq, for Lq = Lk, Lq < Lk
                        and Lq > Lk (bottom-right alignment).
  sequences_independent a packed batch equals each sequence run alone through
                        the unmasked oracle (non-causal) and row-wise prefix
                        checks (causal): keys and queries of other sequences
                        never leak in.
  torch_masked_jvp      torch.func.jvp of softmax(s q k^T + mask) v in fp64
                        with -inf on invisible keys, rows with a visible key.
  empty_rows            rows with no visible key: O = tO = 0, lse = -inf.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


def _rel(a, b):
    den = max(float(np.max(np.abs(b))), 1e-300)
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b)))) / den


def _packed(rng, H, lq, lk, d):
    Tq, Tk = sum(lq), sum(lk)
    x = [rng.standard_normal((H, Tq if i in (0, 3) else Tk, d)) for i in range(6)]
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int64)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int64)
    return x, cu_q, cu_k


def prefix_property(f):
    rng = np.random.default_rng(21)
    worst = 0.0
    for Lq, Lk in ((7, 7), (5, 9), (9, 5)):
        x, cq, ck = _packed(rng, 2, [Lq], [Lk], 4)
        o, to, lse = f(*x, 0.6, cq, ck, True)
        for i in range(Lq):
            n = min(Lk, i + Lk - Lq + 1)
            if n <= 0:
                continue
            r = oracle.attn_jvp(x[0][:, i:i + 1], x[1][:, :n], x[2][:, :n], x[3][:, i:i + 1], x[4][:, :n],
                                x[5][:, :n], 0.6)
            worst = max(worst, _rel(o[:, i], r[0][:, 0]), _rel(to[:, i], r[1][:, 0]), _rel(lse[:, i], r[2][:, 0]))
    return worst < 1e-12, f"worst rel err {worst:.2e}"


def sequences_independent(f):
    rng = np.random.default_rng(22)
    lq, lk = [3, 6, 1, 5], [4, 2, 7, 5]
    x, cq, ck = _packed(rng, 2, lq, lk, 4)
    worst = 0.0
    o, to, lse = f(*x, 0.4, cq, ck, False)
    for b in range(len(lq)):
        qs, ks = slice(cq[b], cq[b + 1]), slice(ck[b], ck[b + 1])
        r = oracle.attn_jvp(x[0][:, qs], x[1][:, ks], x[2][:, ks], x[3][:, qs], x[4][:, ks], x[5][:, ks], 0.4)
        worst = max(worst, _rel(o[:, qs], r[0]), _rel(to[:, qs], r[1]), _rel(lse[:, qs], r[2]))
    oc, toc, lsec = f(*x, 0.4, cq, ck, True)
    for b in range(len(lq)):
        Lq, Lk = lq[b], lk[b]
        for i in range(Lq):
            n = min(Lk, i + Lk - Lq + 1)
            rr = cq[b] + i
            if n <= 0:
                continue
            r = oracle.attn_jvp(x[0][:, rr:rr + 1], x[1][:, ck[b]:ck[b] + n], x[2][:, ck[b]:ck[b] + n],
                                x[3][:, rr:rr + 1], x[4][:, ck[b]:ck[b] + n], x[5][:, ck[b]:ck[b] + n], 0.4)
            worst = max(worst, _rel(oc[:, rr], r[0][:, 0]), _rel(toc[:, rr], r[1][:, 0]))
    return worst < 1e-12, f"worst rel err {worst:.2e}"


def torch_masked_jvp(f):
    rng = np.random.default_rng(23)
    lq, lk = [6, 4], [8, 3]
    x, cq, ck = _packed(rng, 2, lq, lk, 5)
    s = 0.45
    o, to, lse = f(*x, s, cq, ck, True)
    worst = 0.0
    for b in range(2):
        qs, ks = slice(cq[b], cq[b + 1]), slice(ck[b], ck[b + 1])
        Lq, Lk = lq[b], lk[b]
        t = [torch.tensor(a[:, qs] if i in (0, 3) else a[:, ks]) for i, a in enumerate(x)]
        i_idx = torch.arange(Lq)[:, None]
        j_idx = torch.arange(Lk)[None, :]
        mask = torch.where(j_idx <= i_idx + (Lk - Lq), 0.0, float("-inf")).double()

        def attn(q, k, v):
            return torch.softmax(s * q @ k.mT + mask, dim=-1) @ v

        ro, rto = torch.func.jvp(attn, (t[0], t[1], t[2]), (t[3], t[4], t[5]))
        rows = [i for i in range(Lq) if i + Lk - Lq >= 0]
        worst = max(worst, _rel(o[:, qs][:, rows], ro[:, rows].numpy()), _rel(to[:, qs][:, rows], rto[:, rows].numpy()))
    return worst < 1e-12, f"worst rel err {worst:.2e}"


def empty_rows(f):
    rng = np.random.default_rng(24)
    x, cq, ck = _packed(rng, 2, [6], [2], 3)  # causal, Lq > Lk: rows 0..3 see no key
    o, to, lse = f(*x, 0.5, cq, ck, True)
    ok = np.all(o[:, :4] == 0.0) and np.all(to[:, :4] == 0.0) and np.all(np.isneginf(lse[:, :4]))
    ok = ok and np.all(np.isfinite(lse[:, 4:])) and np.any(o[:, 4:] != 0.0)
    return bool(ok), "empty rows zero with lse = -inf; other rows finite" if ok else "empty-row rule broken"


ALL_PINS = {fn.__name__: fn for fn in (prefix_property, sequences_independent, torch_masked_jvp, empty_rows)}


def run_all(f):
    out = {}
    for name, fn in ALL_PINS.items():
        try:
            out[name] = fn(f)
        except Exception as e:
            out[name] = (False, f"raised {type(e).__name__}: {e}")
    return out
