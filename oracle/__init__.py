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

``attn_jvp_bwd_oracle.c`` is the backward counterpart: the gradients of
L = <dO, O> + <dtO, tO> with respect to Q, K, V, tQ, tK, tV, written as the
chain rule through the forward definition's steps in reverse order (the pages
describe the forward only; this is the plain definition of its gradient).
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
_BWD_SRC = os.path.join(_HERE, "attn_jvp_bwd_oracle.c")
_BWD_LIB = os.path.join(_HERE, "liboracle_bwd.so")
_MSK_SRC = os.path.join(_HERE, "attn_jvp_masked_oracle.c")
_MSK_LIB = os.path.join(_HERE, "liboracle_masked.so")
_BMSK_SRC = os.path.join(_HERE, "attn_jvp_bwd_masked_oracle.c")
_BMSK_LIB = os.path.join(_HERE, "liboracle_bwd_masked.so")
_lock = threading.Lock()
_lib = None
_bwd_lib = None
_msk_lib = None
_bmsk_lib = None


def _compile(src: str, lib: str, force: bool) -> str:
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, lib)
    return lib


def build(force: bool = False) -> str:
    """Compile the oracles to ``oracle/liboracle.so`` (forward) and
    ``oracle/liboracle_bwd.so`` (backward) with gcc -O2 and OpenMP.

    No -ffast-math: the oracle keeps IEEE fp64 semantics.
    """
    _compile(_BWD_SRC, _BWD_LIB, force)
    _compile(_MSK_SRC, _MSK_LIB, force)
    _compile(_BMSK_SRC, _BMSK_LIB, force)
    return _compile(_SRC, _LIB, force)


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


def bwd_source_text() -> str:
    with open(_BWD_SRC) as f:
        return f.read()


def masked_source_text() -> str:
    with open(_MSK_SRC) as f:
        return f.read()


def bwd_masked_source_text() -> str:
    with open(_BMSK_SRC) as f:
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


def _bind_bwd(path: str):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int64)
    lib.oracle_attn_jvp_bwd_f64.argtypes = ([dp] * 14 + [ctypes.c_int64] * 4 + [ctypes.c_double]
                                            + [ip, ctypes.c_int64, ip, ctypes.c_int64])
    lib.oracle_attn_jvp_bwd_f64.restype = ctypes.c_int
    return lib


def _get_bwd():
    global _bwd_lib
    with _lock:
        if _bwd_lib is None:
            build()
            _bwd_lib = _bind_bwd(_BWD_LIB)
        return _bwd_lib


def _bind_masked(path: str):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int64)
    lib.oracle_attn_jvp_masked_f64.argtypes = ([dp] * 9 + [ctypes.c_int64] * 4 + [ctypes.c_double, ip, ip,
                                                                               ctypes.c_int64, ctypes.c_int])
    lib.oracle_attn_jvp_masked_f64.restype = ctypes.c_int
    return lib


def _get_masked():
    global _msk_lib
    with _lock:
        if _msk_lib is None:
            build()
            _msk_lib = _bind_masked(_MSK_LIB)
        return _msk_lib


def load_masked_variant(path: str):
    """ctypes handle of a separately compiled masked-oracle build."""
    return _bind_masked(path)


def _bind_bwd_masked(path: str):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int64)
    lib.oracle_attn_jvp_bwd_masked_f64.argtypes = ([dp] * 14 + [ctypes.c_int64] * 4 + [ctypes.c_double]
                                                   + [ip, ip, ctypes.c_int64, ctypes.c_int]
                                                   + [ip, ctypes.c_int64, ip, ctypes.c_int64])
    lib.oracle_attn_jvp_bwd_masked_f64.restype = ctypes.c_int
    return lib


def _get_bwd_masked():
    global _bmsk_lib
    with _lock:
        if _bmsk_lib is None:
            build()
            _bmsk_lib = _bind_bwd_masked(_BMSK_LIB)
        return _bmsk_lib


def load_bwd_masked_variant(path: str):
    """ctypes handle of a separately compiled masked-backward-oracle build."""
    return _bind_bwd_masked(path)


def load_bwd_variant(path: str):
    """ctypes handle of a separately compiled backward-oracle build."""
    return _bind_bwd(path)


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


def attn_jvp_bwd(q, k, v, tq, tk, tv, dout, dtout, scale: float, qrows=None, krows=None, lib=None):
    """Gradients of L = <dout, O> + <dtout, tO> with respect to q, k, v, tq,
    tk, tv (O, tO as ``attn_jvp`` defines them), in fp64.

    Inputs [..., L, d] (leading dims = batch*heads; any float dtype, widened
    exactly).  ``qrows`` / ``krows``: optional lists of query rows / keys whose
    gradients are wanted (default: all); key-side sums always run over every
    query row.  Returns a dict of fp64 numpy arrays: dq, dtq [..., nq, d] and
    dk, dv, dtk, dtv [..., nk, d].
    """
    q, k, v, tq, tk, tv, dout, dtout = (_f64(x) for x in (q, k, v, tq, tk, tv, dout, dtout))
    lead = q.shape[:-2]
    Lq, d = q.shape[-2], q.shape[-1]
    Lk = k.shape[-2]
    for x, L in ((tq, Lq), (dout, Lq), (dtout, Lq), (k, Lk), (v, Lk), (tk, Lk), (tv, Lk)):
        if x.shape != tuple(lead) + (L, d):
            raise ValueError(f"shape mismatch: {x.shape} vs {tuple(lead) + (L, d)}")
    BH = int(np.prod(lead)) if lead else 1
    qr = None if qrows is None else np.ascontiguousarray(np.asarray(qrows, dtype=np.int64))
    kr = None if krows is None else np.ascontiguousarray(np.asarray(krows, dtype=np.int64))
    nq = Lq if qr is None else len(qr)
    nk = Lk if kr is None else len(kr)
    out = {n: np.zeros(tuple(lead) + (nq, d)) for n in ("dq", "dtq")}
    out.update({n: np.zeros(tuple(lead) + (nk, d)) for n in ("dk", "dv", "dtk", "dtv")})
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int64)
    ptr = lambda a: a.ctypes.data_as(dp)  # noqa: E731
    iptr = lambda a: None if a is None else a.ctypes.data_as(ip)  # noqa: E731
    handle = lib if lib is not None else _get_bwd()
    rc = handle.oracle_attn_jvp_bwd_f64(ptr(q), ptr(k), ptr(v), ptr(tq), ptr(tk), ptr(tv), ptr(dout), ptr(dtout),
                                        ptr(out["dq"]), ptr(out["dk"]), ptr(out["dv"]), ptr(out["dtq"]),
                                        ptr(out["dtk"]), ptr(out["dtv"]), BH, Lq, Lk, d, float(scale),
                                        iptr(qr), nq, iptr(kr), nk)
    if rc != 0:
        raise RuntimeError(f"oracle_attn_jvp_bwd_f64 failed with {rc}")
    return out


def attn_jvp_packed(q, k, v, tq, tk, tv, scale: float, cu_q, cu_k, causal: bool, lib=None):
    """Packed (variable-length) attention + JVP, optionally causal.

    q, tq: [H, Tq, d]; k, v, tk, tv: [H, Tk, d]; cu_q, cu_k: cumulative
    sequence starts (length nseq + 1, first 0, last Tq / Tk).  Causal means
    key j of a sequence is visible to its query row i iff j <= i + (Lk - Lq).
    Rows with no visible key give O = tO = 0, lse = -inf.  Returns fp64 numpy
    (O [H, Tq, d], tO [H, Tq, d], lse [H, Tq]).
    """
    q, k, v, tq, tk, tv = (_f64(x) for x in (q, k, v, tq, tk, tv))
    H, Tq, d = q.shape
    Tk = k.shape[1]
    cq = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int64))
    ck = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int64))
    o = np.empty((H, Tq, d))
    to = np.empty_like(o)
    lse = np.empty((H, Tq))
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int64)
    ptr = lambda a: a.ctypes.data_as(dp)  # noqa: E731
    handle = lib if lib is not None else _get_masked()
    rc = handle.oracle_attn_jvp_masked_f64(ptr(q), ptr(k), ptr(v), ptr(tq), ptr(tk), ptr(tv), ptr(o), ptr(to),
                                           ptr(lse), H, Tq, Tk, d, float(scale), cq.ctypes.data_as(ip),
                                           ck.ctypes.data_as(ip), len(cq) - 1, int(bool(causal)))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_jvp_masked_f64 failed with {rc}")
    return o, to, lse


def attn_jvp_causal(q, k, v, tq, tk, tv, scale: float, lib=None):
    """Causal attention + JVP for dense [..., L, d] tensors (one sequence per
    leading index; bottom-right aligned when Lq != Lk)."""
    q, k, v, tq, tk, tv = (_f64(x) for x in (q, k, v, tq, tk, tv))
    lead = q.shape[:-2]
    Lq, d = q.shape[-2], q.shape[-1]
    Lk = k.shape[-2]
    BH = int(np.prod(lead)) if lead else 1
    f = lambda x, L: x.reshape(BH, L, d)  # noqa: E731
    o, to, lse = attn_jvp_packed(f(q, Lq), f(k, Lk), f(v, Lk), f(tq, Lq), f(tk, Lk), f(tv, Lk), scale,
                                 [0, Lq], [0, Lk], True, lib=lib)
    return o.reshape(q.shape), to.reshape(q.shape), lse.reshape(tuple(lead) + (Lq,))


def attn_jvp_bwd_packed(q, k, v, tq, tk, tv, dout, dtout, scale: float, cu_q, cu_k, causal: bool,
                        qrows=None, krows=None, lib=None):
    """Gradients of L = <dout, O> + <dtout, tO> for packed (variable-length),
    optionally causal attention + JVP (O, tO as ``attn_jvp_packed`` defines
    them), in fp64.

    q, tq, dout, dtout: [H, Tq, d]; k, v, tk, tv: [H, Tk, d]; cu_q, cu_k as
    for ``attn_jvp_packed``.  ``qrows`` / ``krows``: optional packed query rows
    / key rows whose gradients are wanted (default: all); key-side sums run
    over every query row of the key's sequence.  Returns a dict of fp64 numpy
    arrays: dq, dtq [H, nq, d] and dk, dv, dtk, dtv [H, nk, d].
    """
    q, k, v, tq, tk, tv, dout, dtout = (_f64(x) for x in (q, k, v, tq, tk, tv, dout, dtout))
    H, Tq, d = q.shape
    Tk = k.shape[1]
    for x, T in ((tq, Tq), (dout, Tq), (dtout, Tq), (k, Tk), (v, Tk), (tk, Tk), (tv, Tk)):
        if x.shape != (H, T, d):
            raise ValueError(f"shape mismatch: {x.shape} vs {(H, T, d)}")
    cq = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int64))
    ck = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int64))
    qr = None if qrows is None else np.ascontiguousarray(np.asarray(qrows, dtype=np.int64))
    kr = None if krows is None else np.ascontiguousarray(np.asarray(krows, dtype=np.int64))
    nq = Tq if qr is None else len(qr)
    nk = Tk if kr is None else len(kr)
    out = {n: np.zeros((H, nq, d)) for n in ("dq", "dtq")}
    out.update({n: np.zeros((H, nk, d)) for n in ("dk", "dv", "dtk", "dtv")})
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int64)
    ptr = lambda a: a.ctypes.data_as(dp)  # noqa: E731
    iptr = lambda a: None if a is None else a.ctypes.data_as(ip)  # noqa: E731
    handle = lib if lib is not None else _get_bwd_masked()
    rc = handle.oracle_attn_jvp_bwd_masked_f64(ptr(q), ptr(k), ptr(v), ptr(tq), ptr(tk), ptr(tv), ptr(dout),
                                               ptr(dtout), ptr(out["dq"]), ptr(out["dk"]), ptr(out["dv"]),
                                               ptr(out["dtq"]), ptr(out["dtk"]), ptr(out["dtv"]), H, Tq, Tk, d,
                                               float(scale), iptr(cq), iptr(ck), len(cq) - 1, int(bool(causal)),
                                               iptr(qr), nq, iptr(kr), nk)
    if rc != 0:
        raise RuntimeError(f"oracle_attn_jvp_bwd_masked_f64 failed with {rc}")
    return out


def attn_jvp_bwd_causal(q, k, v, tq, tk, tv, dout, dtout, scale: float, qrows=None, krows=None, lib=None):
    """Causal backward for dense [..., L, d] tensors (one sequence per leading
    index; bottom-right aligned when Lq != Lk).  ``qrows`` / ``krows`` index
    rows within one sequence (the same rows for every leading index).
    Returns dq, dtq [..., nq, d] and dk, dv, dtk, dtv [..., nk, d]."""
    q, k, v, tq, tk, tv, dout, dtout = (_f64(x) for x in (q, k, v, tq, tk, tv, dout, dtout))
    lead = q.shape[:-2]
    Lq, d = q.shape[-2], q.shape[-1]
    Lk = k.shape[-2]
    BH = int(np.prod(lead)) if lead else 1
    f = lambda x, L: x.reshape(BH, L, d)  # noqa: E731
    g = attn_jvp_bwd_packed(f(q, Lq), f(k, Lk), f(v, Lk), f(tq, Lq), f(tk, Lk), f(tv, Lk), f(dout, Lq),
                            f(dtout, Lq), scale, [0, Lq], [0, Lk], True, qrows=qrows, krows=krows, lib=lib)
    nq = Lq if qrows is None else len(qrows)
    nk = Lk if krows is None else len(krows)
    return {n: a.reshape(tuple(lead) + ((nq if n in ("dq", "dtq") else nk), d)) for n, a in g.items()}
