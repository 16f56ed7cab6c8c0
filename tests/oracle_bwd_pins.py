"""Checks that pin the fp64 backward oracle to facts other than itself.

Each pin takes a backward callable
``g(q, k, v, tq, tk, tv, dout, dtout, scale, qrows=None, krows=None) -> dict``
(dq, dk, dv, dtq, dtk, dtv as fp64 arrays) and returns (ok, detail).  The
gradients are those of L = <dout, O> + <dtout, tO>, O and tO being attention
and its JVP.  A plausible slip anywhere in the oracle (a dropped chain-rule
term, a wrong sign, a swapped operand, a missing scale) fails at least one
pin; tests/test_oracle_bwd_mutants.py plants such slips and checks that.

What pins what:
  finite_difference     <grad, e> equals the central difference of L (the
                        forward oracle, itself pinned) along a random e, for
                        each of the six inputs; self- and cross-attention.
  torch_reverse_jvp     all six gradients equal torch.autograd through
                        torch.func.jvp of the same attention (fp64).
  standard_backward     dtout = 0: dq, dk, dv are the ordinary attention
                        gradients (torch autograd of softmax(s q k^T) v) and
                        dtq, dtk, dtv vanish.
  tangent_independence  tO is linear in the tangent, so dtq, dtk, dtv do not
                        depend on (tq, tk, tv).
  cotangent_linearity   every gradient is linear in (dout, dtout).
  dtv_closed_form       dtv = softmax(s q k^T)^T dtout (library softmax).
  subsets               gradients of listed query rows / keys equal the rows
                        of the full result.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

NAMES = ("dq", "dk", "dv", "dtq", "dtk", "dtv")


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = max(float(np.max(np.abs(b))), 1e-300)
    return float(np.max(np.abs(a - b))) / den


def _inputs(rng, BH=2, Lq=5, Lk=7, d=4):
    x = {n: rng.standard_normal((BH, Lq if n in ("q", "tq", "dout", "dtout") else Lk, d))
         for n in ("q", "k", "v", "tq", "tk", "tv", "dout", "dtout")}
    return x


def _call(g, x, s, **kw):
    return g(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], x["dout"], x["dtout"], s, **kw)


def _loss(x, s):
    o, to, _ = oracle.attn_jvp(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], s)
    return float(np.sum(o * x["dout"]) + np.sum(to * x["dtout"]))


def finite_difference(g):
    rng = np.random.default_rng(11)
    worst = 0.0
    for shape in ((2, 5, 7, 4), (1, 9, 3, 6), (1, 4, 4, 8)):
        x = _inputs(rng, *shape)
        s = 0.6
        grads = _call(g, x, s)
        eps = 1e-6
        for name, gname in zip(("q", "k", "v", "tq", "tk", "tv"), NAMES):
            e = rng.standard_normal(x[name].shape)
            xp = dict(x)
            xm = dict(x)
            xp[name] = x[name] + eps * e
            xm[name] = x[name] - eps * e
            fd = (_loss(xp, s) - _loss(xm, s)) / (2 * eps)
            an = float(np.sum(grads[gname] * e))
            scale = float(np.linalg.norm(grads[gname]) * np.linalg.norm(e)) + 1e-30
            worst = max(worst, abs(fd - an) / scale)
    return worst < 1e-7, f"worst |fd - <g,e>| / (|g||e|) = {worst:.2e}"


def _torch_grads(x, s):
    t = {n: torch.tensor(x[n], dtype=torch.float64, requires_grad=n in ("q", "k", "v", "tq", "tk", "tv"))
         for n in x}

    def attn(q, k, v):
        return torch.softmax(s * q @ k.mT, dim=-1) @ v

    o, to = torch.func.jvp(attn, (t["q"], t["k"], t["v"]), (t["tq"], t["tk"], t["tv"]))
    loss = (o * t["dout"]).sum() + (to * t["dtout"]).sum()
    gr = torch.autograd.grad(loss, [t[n] for n in ("q", "k", "v", "tq", "tk", "tv")])
    return dict(zip(NAMES, (a.numpy() for a in gr)))


def torch_reverse_jvp(g):
    rng = np.random.default_rng(12)
    worst = 0.0
    for shape in ((2, 6, 6, 5), (3, 4, 9, 3)):
        x = _inputs(rng, *shape)
        got = _call(g, x, 0.45)
        ref = _torch_grads(x, 0.45)
        worst = max(worst, max(_rel(got[n], ref[n]) for n in NAMES))
    return worst < 1e-10, f"worst rel err {worst:.2e}"


def standard_backward(g):
    rng = np.random.default_rng(13)
    x = _inputs(rng, 2, 6, 8, 4)
    x["dtout"] = np.zeros_like(x["dtout"])
    s = 0.8
    got = _call(g, x, s)
    t = {n: torch.tensor(x[n], dtype=torch.float64, requires_grad=n in ("q", "k", "v")) for n in ("q", "k", "v")}
    o = torch.softmax(s * t["q"] @ t["k"].mT, dim=-1) @ t["v"]
    gq, gk, gv = torch.autograd.grad((o * torch.tensor(x["dout"])).sum(), [t["q"], t["k"], t["v"]])
    err = max(_rel(got["dq"], gq.numpy()), _rel(got["dk"], gk.numpy()), _rel(got["dv"], gv.numpy()))
    zero = all(np.all(got[n] == 0.0) for n in ("dtq", "dtk", "dtv"))
    return err < 1e-12 and zero, f"rel err {err:.2e}, tangent grads zero: {zero}"


def tangent_independence(g):
    rng = np.random.default_rng(14)
    x = _inputs(rng, 2, 5, 7, 4)
    a = _call(g, x, 0.5)
    y = dict(x)
    for n in ("tq", "tk", "tv"):
        y[n] = rng.standard_normal(x[n].shape) * 3.0
    b = _call(g, y, 0.5)
    err = max(_rel(b[n], a[n]) for n in ("dtq", "dtk", "dtv"))
    moved = _rel(b["dq"], a["dq"]) > 1e-3  # the primal gradients do depend on the tangent
    return err < 1e-12 and moved, f"rel change of tangent grads {err:.2e}, primal grads moved: {moved}"


def cotangent_linearity(g):
    rng = np.random.default_rng(15)
    x = _inputs(rng, 1, 6, 5, 4)
    y = dict(x)
    y["dout"] = rng.standard_normal(x["dout"].shape)
    y["dtout"] = rng.standard_normal(x["dtout"].shape)
    z = dict(x)
    z["dout"] = 2.0 * x["dout"] - 0.5 * y["dout"]
    z["dtout"] = 2.0 * x["dtout"] - 0.5 * y["dtout"]
    a, b, c = _call(g, x, 0.7), _call(g, y, 0.7), _call(g, z, 0.7)
    err = max(_rel(c[n], 2.0 * a[n] - 0.5 * b[n]) for n in NAMES)
    return err < 1e-12, f"rel err {err:.2e}"


def dtv_closed_form(g):
    rng = np.random.default_rng(16)
    x = _inputs(rng, 2, 7, 5, 3)
    s = 0.9
    got = _call(g, x, s)
    p = torch.softmax(s * torch.tensor(x["q"]) @ torch.tensor(x["k"]).mT, dim=-1)
    ref = (p.mT @ torch.tensor(x["dtout"])).numpy()
    err = _rel(got["dtv"], ref)
    return err < 1e-12, f"rel err {err:.2e}"


def subsets(g):
    rng = np.random.default_rng(17)
    x = _inputs(rng, 2, 9, 11, 4)
    full = _call(g, x, 0.5)
    qr, kr = [7, 0, 3], [10, 2]
    sub = _call(g, x, 0.5, qrows=qr, krows=kr)
    ok = all(np.array_equal(sub[n], full[n][:, qr]) for n in ("dq", "dtq"))
    ok = ok and all(np.array_equal(sub[n], full[n][:, kr]) for n in ("dk", "dv", "dtk", "dtv"))
    return ok, "subset rows equal the full result's rows" if ok else "subset mismatch"


ALL_PINS = {f.__name__: f for f in (finite_difference, torch_reverse_jvp, standard_backward, tangent_independence,
                                     cotangent_linearity, dtv_closed_form, subsets)}


def run_all(g):
    out = {}
    for name, fn in ALL_PINS.items():
        try:
            out[name] = fn(g)
        except Exception as e:  # a broken oracle may also fail by raising
            out[name] = (False, f"raised {type(e).__name__}: {e}")
    return out
