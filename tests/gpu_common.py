"""Shared helpers for the GPU parity tests: run the CUDA path through the C
ABI binding, run the fp64 oracle on the same inputs (whole tensors or sampled
rows), and measure max|err| / max|ref|."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from attention_forward_mode_b200 import attn_jvp
from attention_forward_mode_b200.workloads import Workload, make_inputs, sample_rows

# acceptance bounds on max|err| / max|ref| against the fp64 oracle
TOL = {"bf16": {"o": 1e-2, "to": 2e-2, "lse": 1e-3}, "f32": {"o": 1e-4, "to": 1e-4, "lse": 1e-5}}


def max_rel(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.max(np.abs(ref)))
    if den == 0.0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got - ref))) / den


def run_cuda(inp: dict, scale: float):
    o, to, lse = attn_jvp(inp["q"], inp["k"], inp["v"], inp["tq"], inp["tk"], inp["tv"], scale)
    torch.cuda.synchronize()
    return o, to, lse


def gpu_inputs(w: Workload, seed: int = 0):
    return make_inputs(w, seed=seed, device="cuda")


def flat(x):
    return x.reshape(-1, x.shape[-2], x.shape[-1])


def compare_full(w: Workload, inp: dict, out) -> dict:
    """Oracle on every row of every head (small workloads)."""
    cpu = {n: t.cpu() for n, t in inp.items()}
    ro, rto, rlse = oracle.attn_jvp(cpu["q"], cpu["k"], cpu["v"], cpu["tq"], cpu["tk"], cpu["tv"], w.scale)
    o, to, lse = (t.float().cpu().numpy() for t in out)
    return {"o": max_rel(o, ro), "to": max_rel(to, rto), "lse": max_rel(lse, rlse)}


def compare_rows(w: Workload, inp: dict, out, heads, n_rows: int, seed: int = 0, rows=None) -> dict:
    """Oracle on sampled query rows of sampled heads (rows are independent,
    so this is the full oracle restricted to them).  ``rows``: an explicit
    row list instead of the seeded sample."""
    if rows is None:
        rows = sample_rows(w.Lq, n_rows, seed=seed)
    fl = {n: flat(t) for n, t in inp.items()}
    got_o, got_to, got_l = [], [], []
    ref_o, ref_to, ref_l = [], [], []
    lse_flat = out[2].reshape(-1, w.Lq)
    idx = torch.tensor(rows, device=out[0].device)
    for h in heads:
        q = fl["q"][h].index_select(0, idx).cpu()
        tq = fl["tq"][h].index_select(0, idx).cpu()
        k, v, tk, tv = (fl[n][h].cpu() for n in ("k", "v", "tk", "tv"))
        r = oracle.attn_jvp(q[None], k[None], v[None], tq[None], tk[None], tv[None], w.scale)
        ref_o.append(r[0][0]); ref_to.append(r[1][0]); ref_l.append(r[2][0])
        got_o.append(flat(out[0])[h].index_select(0, idx).float().cpu().numpy())
        got_to.append(flat(out[1])[h].index_select(0, idx).float().cpu().numpy())
        got_l.append(lse_flat[h].index_select(0, idx).cpu().numpy())
    return {"o": max_rel(np.stack(got_o), np.stack(ref_o)),
            "to": max_rel(np.stack(got_to), np.stack(ref_to)),
            "lse": max_rel(np.stack(got_l), np.stack(ref_l)),
            "rows": len(rows), "heads": list(heads)}


def assert_within(err: dict, dtype: str, what: str):
    tol = TOL[dtype]
    for key in ("o", "to", "lse"):
        assert err[key] <= tol[key], f"{what}: {key} max-rel error {err[key]:.3e} > {tol[key]:.0e} ({err})"
