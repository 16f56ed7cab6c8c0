"""Checks that pin the fp64 oracle to facts other than itself.

Each pin takes an oracle callable ``f(q, k, v, tq, tk, tv, scale) -> (O, tO, lse)``
working on fp64 arrays of shape [BH, L, d] and returns (ok, detail).  The
pins are chosen so that a plausible slip anywhere in the oracle (a dropped
term, a wrong sign, a transposed or swapped operand, a missing scale or
normalisation) fails at least one of them; tests/test_oracle_mutants.py
plants such slips in copies of the oracle and checks exactly that.

What pins what:
  two_key_closed_form  Lk = 2, d = 1: P is a logistic function of the score
                       gap and tO follows by hand differentiation.
  single_key           Lk = 1: softmax is 1, so O = V, tO = tV, lse = s q.k.
  primal_vs_torch      O and lse equal torch.softmax / torch.logsumexp (fp64).
  finite_difference    tO equals the central difference of O along the
                       tangent, eps = 1e-6 (fp64; O(eps^2) truncation).
  torch_func_jvp       tO equals torch.func.jvp of the same attention (fp64).
  linearity            tO is linear in the tangent (tQ, tK, tV).
  zero_tangent         tO is exactly 0 for a zero tangent.
  shift_invariance     tQ = 0, tK = the same vector c for every key, tV = 0:
                       every score of a row moves by the same amount, softmax
                       is unchanged, so tO = 0.
  ptv_term             tQ = tK = 0: tO = attention(Q, K, tV).
  key_permutation      permuting the keys (with their V, tK, tV) changes
                       nothing; permuting query rows permutes the outputs.
"""
from __future__ import annotations

import math

import numpy as np
import torch


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = max(float(np.max(np.abs(b))), 1e-300)
    return float(np.max(np.abs(a - b))) / den


def _rand(rng, *shape, std=1.0):
    return rng.standard_normal(shape) * std


def _inputs(rng, BH=2, Lq=5, Lk=7, d=4, std=1.0, tstd=1.0):
    q = _rand(rng, BH, Lq, d, std=std)
    k = _rand(rng, BH, Lk, d, std=std)
    v = _rand(rng, BH, Lk, d)
    tq = _rand(rng, BH, Lq, d, std=tstd)
    tk = _rand(rng, BH, Lk, d, std=tstd)
    tv = _rand(rng, BH, Lk, d, std=tstd)
    return q, k, v, tq, tk, tv


def pin_two_key_closed_form(f):
    rng = np.random.default_rng(11)
    s = 0.7
    q, k, v, tq, tk, tv = _inputs(rng, BH=1, Lq=3, Lk=2, d=1)
    O, tO, lse = f(q, k, v, tq, tk, tv, s)
    worst = 0.0
    for i in range(3):
        qi, tqi = q[0, i, 0], tq[0, i, 0]
        k1, k2 = k[0, 0, 0], k[0, 1, 0]
        v1, v2 = v[0, 0, 0], v[0, 1, 0]
        tk1, tk2 = tk[0, 0, 0], tk[0, 1, 0]
        tv1, tv2 = tv[0, 0, 0], tv[0, 1, 0]
        gap = s * qi * (k1 - k2)
        p1 = 1.0 / (1.0 + math.exp(-gap))
        p2 = 1.0 - p1
        o = p1 * v1 + p2 * v2
        dgap = s * (tqi * (k1 - k2) + qi * (tk1 - tk2))
        dp1 = p1 * p2 * dgap
        to = dp1 * (v1 - v2) + p1 * tv1 + p2 * tv2
        l = max(s * qi * k1, s * qi * k2) + math.log(
            math.exp(s * qi * k1 - max(s * qi * k1, s * qi * k2))
            + math.exp(s * qi * k2 - max(s * qi * k1, s * qi * k2)))
        worst = max(worst, abs(O[0, i, 0] - o), abs(tO[0, i, 0] - to), abs(lse[0, i] - l))
    return worst < 1e-13, f"max abs err {worst:.3e}"


def pin_single_key(f):
    rng = np.random.default_rng(12)
    s = 0.3
    q, k, v, tq, tk, tv = _inputs(rng, BH=2, Lq=4, Lk=1, d=6)
    O, tO, lse = f(q, k, v, tq, tk, tv, s)
    e1 = _rel(O, np.broadcast_to(v, O.shape))
    e2 = _rel(tO, np.broadcast_to(tv, tO.shape))
    ref_lse = s * np.einsum("hid,hjd->hij", q, k)[..., 0]
    e3 = _rel(lse, ref_lse)
    return max(e1, e2, e3) < 1e-14, f"O {e1:.2e} tO {e2:.2e} lse {e3:.2e}"


def pin_primal_vs_torch(f):
    rng = np.random.default_rng(13)
    s = 0.45
    q, k, v, tq, tk, tv = _inputs(rng, BH=3, Lq=9, Lk=13, d=5, std=1.5)
    O, _, lse = f(q, k, v, tq, tk, tv, s)
    Qt, Kt, Vt = (torch.from_numpy(x) for x in (q, k, v))
    S = s * Qt @ Kt.transpose(-1, -2)
    ref_o = torch.softmax(S, dim=-1) @ Vt
    ref_lse = torch.logsumexp(S, dim=-1)
    e1, e2 = _rel(O, ref_o.numpy()), _rel(lse, ref_lse.numpy())
    return max(e1, e2) < 1e-12, f"O {e1:.2e} lse {e2:.2e}"


def pin_finite_difference(f):
    rng = np.random.default_rng(14)
    s = 0.6
    q, k, v, tq, tk, tv = _inputs(rng, BH=2, Lq=6, Lk=11, d=4)
    _, tO, _ = f(q, k, v, tq, tk, tv, s)
    eps = 1e-6
    zeros = [np.zeros_like(x) for x in (tq, tk, tv)]
    Op, _, _ = f(q + eps * tq, k + eps * tk, v + eps * tv, *zeros, s)
    Om, _, _ = f(q - eps * tq, k - eps * tk, v - eps * tv, *zeros, s)
    fd = (Op - Om) / (2 * eps)
    e = _rel(tO, fd)
    return e < 1e-7, f"rel err vs central difference {e:.2e}"


def pin_torch_func_jvp(f):
    rng = np.random.default_rng(15)
    s = 0.5
    q, k, v, tq, tk, tv = _inputs(rng, BH=2, Lq=7, Lk=10, d=3)
    _, tO, _ = f(q, k, v, tq, tk, tv, s)

    def attn(a, b, c):
        return torch.softmax(s * a @ b.transpose(-1, -2), dim=-1) @ c

    T = [torch.from_numpy(x) for x in (q, k, v, tq, tk, tv)]
    _, ref = torch.func.jvp(attn, tuple(T[:3]), tuple(T[3:]))
    e = _rel(tO, ref.numpy())
    return e < 1e-12, f"rel err vs torch.func.jvp {e:.2e}"


def pin_linearity(f):
    rng = np.random.default_rng(16)
    s = 0.4
    q, k, v, a_q, a_k, a_v = _inputs(rng, BH=1, Lq=5, Lk=8, d=4)
    _, _, _, b_q, b_k, b_v = _inputs(rng, BH=1, Lq=5, Lk=8, d=4)
    alpha, beta = 0.75, -1.25
    _, ta, _ = f(q, k, v, a_q, a_k, a_v, s)
    _, tb, _ = f(q, k, v, b_q, b_k, b_v, s)
    _, tc, _ = f(q, k, v, alpha * a_q + beta * b_q, alpha * a_k + beta * b_k,
                 alpha * a_v + beta * b_v, s)
    e = _rel(tc, alpha * ta + beta * tb)
    return e < 1e-12, f"rel err {e:.2e}"


def pin_zero_tangent(f):
    rng = np.random.default_rng(17)
    q, k, v, tq, tk, tv = _inputs(rng, BH=2, Lq=4, Lk=6, d=3)
    z = [np.zeros_like(x) for x in (tq, tk, tv)]
    _, tO, _ = f(q, k, v, *z, 0.5)
    return bool(np.all(tO == 0.0)), f"max |tO| {float(np.max(np.abs(tO))):.2e}"


def pin_shift_invariance(f):
    rng = np.random.default_rng(18)
    s = 0.55
    q, k, v, _, _, _ = _inputs(rng, BH=2, Lq=6, Lk=9, d=5)
    c = rng.standard_normal((2, 1, 5))
    tk = np.broadcast_to(c, k.shape).copy()
    _, tO, _ = f(q, k, v, np.zeros_like(q), tk, np.zeros_like(v), s)
    bound = 1e-13 * float(np.max(np.abs(c))) * float(np.max(np.abs(v))) * 10
    m = float(np.max(np.abs(tO)))
    return m <= bound, f"max |tO| {m:.2e} (bound {bound:.1e})"


def pin_ptv_term(f):
    rng = np.random.default_rng(19)
    s = 0.35
    q, k, v, _, _, tv = _inputs(rng, BH=2, Lq=5, Lk=7, d=4)
    _, tO, _ = f(q, k, v, np.zeros_like(q), np.zeros_like(k), tv, s)
    O2, _, _ = f(q, k, tv, np.zeros_like(q), np.zeros_like(k), np.zeros_like(tv), s)
    e = _rel(tO, O2)
    return e < 1e-13, f"rel err {e:.2e}"


def pin_key_permutation(f):
    rng = np.random.default_rng(20)
    s = 0.5
    q, k, v, tq, tk, tv = _inputs(rng, BH=1, Lq=6, Lk=9, d=3)
    O, tO, lse = f(q, k, v, tq, tk, tv, s)
    pk = rng.permutation(9)
    pq = rng.permutation(6)
    O2, tO2, lse2 = f(q[:, pq], k[:, pk], v[:, pk], tq[:, pq], tk[:, pk], tv[:, pk], s)
    e = max(_rel(O2, O[:, pq]), _rel(tO2, tO[:, pq]), _rel(lse2, lse[:, pq]))
    return e < 1e-13, f"rel err {e:.2e}"


ALL_PINS = {
    "two_key_closed_form": pin_two_key_closed_form,
    "single_key": pin_single_key,
    "primal_vs_torch": pin_primal_vs_torch,
    "finite_difference": pin_finite_difference,
    "torch_func_jvp": pin_torch_func_jvp,
    "linearity": pin_linearity,
    "zero_tangent": pin_zero_tangent,
    "shift_invariance": pin_shift_invariance,
    "ptv_term": pin_ptv_term,
    "key_permutation": pin_key_permutation,
}


def run_all(f):
    """{pin name: (ok, detail)} for an oracle callable."""
    out = {}
    for name, pin in ALL_PINS.items():
        try:
            out[name] = pin(f)
        except Exception as exc:  # a broken oracle may also crash a pin
            out[name] = (False, f"raised {type(exc).__name__}: {exc}")
    return out
