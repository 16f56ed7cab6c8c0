"""fp64 CPU oracle for attention + its Jacobian-vector product.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The product path (the CUDA library
under ``attention_forward_mode_b200``) never imports this package, and this
package imports nothing from it.

The arithmetic lives in ``attn_jvp_oracle.c`` (plain loops, fp64, OpenMP over
query rows); this module only compiles it with gcc and marshals numpy arrays.
What it computes: rCM (anthology record LIT-783, §3.2 / App. C) fuses a
FlashAttention-2 forward with its JVP; the oracle is the plain definition --
O = softmax(s Q K^T) V and tO = d/dt O(Q + t tQ, K + t tK, V + t tV) at t = 0,
written as sum_j P_ij (dS_ij - mu_i) V_j + sum_j P_ij tV_j with
dS = s (tQ K^T + Q tK^T) and mu_i = sum_j P_ij dS_ij, plus lse = ln sum_j exp(S_ij).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_jvp_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle to ``oracle/liboracle.so`` (gcc, -O2, OpenMP).

    No -ffast-math: the oracle keeps IEEE fp64 semantics.
    """
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def compile_variant(src_text: str, out_path: str) -> str:
    """Compile an edited copy of the oracle source (used by the tests that
    plant a mistake in the oracle to show the pins catch it)."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           "-o", out_path, c_path, "-lm"])
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _bind(path: str):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_attn_jvp_f64.argtypes = [dp] * 9 + [ctypes.c_int64] * 4 + [ctypes.c_double]
    lib.oracle_attn_jvp_f64.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def _get():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
        return _lib


def load_variant(path: str):
    """ctypes handle of a separately compiled oracle build."""
    return _bind(path)


def num_threads() -> int:
    return int(_get().oracle_num_threads())


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor -> exact fp64 (bf16/fp32 widen exactly)
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def attn_jvp(q, k, v, tq, tk, tv, scale: float, lib=None):
    """O, tO, lse for inputs of shape [..., L, d] (leading dims = batch*heads).

    q, tq: [..., Lq, d]; k, v, tk, tv: [..., Lk, d].  Any float dtype is
    widened exactly to fp64 first.  Returns fp64 numpy arrays
    (O [..., Lq, d], tO [..., Lq, d], lse [..., Lq]).
    """
    q, k, v, tq, tk, tv = (_f64(x) for x in (q, k, v, tq, tk, tv))
    lead = q.shape[:-2]
    Lq, d = q.shape[-2], q.shape[-1]
    Lk = k.shape[-2]
    for x, L in ((tq, Lq), (k, Lk), (v, Lk), (tk, Lk), (tv, Lk)):
        if x.shape != tuple(lead) + (L, d):
            raise ValueError(f"shape mismatch: {x.shape} vs {tuple(lead) + (L, d)}")
    BH = int(np.prod(lead)) if lead else 1
    o = np.empty(tuple(lead) + (Lq, d), dtype=np.float64)
    to = np.empty_like(o)
    lse = np.empty(tuple(lead) + (Lq,), dtype=np.float64)
    dp = ctypes.POINTER(ctypes.c_double)
    ptr = lambda a: a.ctypes.data_as(dp)  # noqa: E731
    handle = lib if lib is not None else _get()
    rc = handle.oracle_attn_jvp_f64(ptr(q), ptr(k), ptr(v), ptr(tq), ptr(tk), ptr(tv),
                                    ptr(o), ptr(to), ptr(lse), BH, Lq, Lk, d, float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_jvp_f64 failed with {rc}")
    return o, to, lse


def attn_jvp_rows(q, k, v, tq, tk, tv, scale: float, heads, rows):
    """Oracle on a subset: for each flattened head index h in ``heads`` and
    query rows ``rows`` (same rows for every listed head).  q-like inputs are
    [BH, Lq, d], k-like [BH, Lk, d] (torch or numpy, any float dtype).
    Rows are independent, so this equals the full oracle restricted to them.
    Returns (O [nh, nr, d], tO [nh, nr, d], lse [nh, nr]).
    """
    outs = []
    for h in heads:
        qs = _f64(q[h][rows]) if not hasattr(q, "detach") else _f64(q[h][list(rows)])
        tqs = _f64(tq[h][rows]) if not hasattr(tq, "detach") else _f64(tq[h][list(rows)])
        outs.append(attn_jvp(qs[None], _f64(k[h])[None], _f64(v[h])[None], tqs[None],
                             _f64(tk[h])[None], _f64(tv[h])[None], scale))
    o = np.concatenate([x[0] for x in outs])
    to = np.concatenate([x[1] for x in outs])
    lse = np.concatenate([x[2] for x in outs])
    return o, to, lse
