"""ctypes binding of the C ABI in ``include/attn_jvp.h``.

Argument marshalling only: shape/dtype/device checks of torch tensors, raw
pointers handed to the library, status codes turned into exceptions.  Every
step of the computation runs in the library's CUDA kernels; there is no other
implementation to fall back to, so a missing library raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattnjvp.so")

AJVP_OK = 0
AJVP_ERR_INVALID_ARG = -1
AJVP_ERR_UNSUPPORTED_DIM = -2
AJVP_ERR_MISALIGNED = -3
AJVP_ERR_UNSUPPORTED_DEVICE = -4
AJVP_ERR_TIMEOUT = -5
AJVP_ERR_CUDA = -6
AJVP_ERR_TOO_LARGE = -7
AJVP_ERR_WORKSPACE = -8
AJVP_ERR_DEVICE_LAYOUT = -9

# every symbol the header declares
EXPORTED = (
    "attn_jvp_fwd", "attn_jvp_fwd_causal", "attn_jvp_fwd_varlen", "attn_jvp_fwd_f32out", "attn_jvp_fwd_stats",
    "attn_jvp_fwd_causal_stats", "attn_jvp_bwd", "attn_jvp_bwd_step", "attn_jvp_bwd_causal",
    "attn_jvp_fwd_varlen_stats", "attn_jvp_bwd_varlen", "attn_jvp_fwd_f32out_causal",
    "attn_jvp_fwd_f32out_varlen", "attn_jvp_bwd_workspace_bytes", "attn_jvp_bwd_workspace_bytes_split",
    "attn_jvp_bwd_key_split_parts", "attn_jvp_fwd_f32", "attn_jvp_fwd_host", "attn_jvp_fwd_host_noalloc",
    "attn_jvp_host_workspace_bytes", "attn_jvp_bwd_host", "attn_jvp_bwd_host_workspace_bytes",
    "attn_jvp_strerror", "attn_jvp_last_cuda_error", "attn_jvp_check_device_status",
    "attn_jvp_set_wait_bound_ns", "attn_jvp_set_persistent_key_tiles", "attn_jvp_set_bwd_pairs",
    "attn_jvp_selftest_wait_timeout",
    "attn_jvp_version",
)

_lock = threading.Lock()
_lib = None


class AttnJvpError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(what)


def load_library(path: str = LIB_PATH):
    """Load (once) and type the shared library.  Raises if it is missing."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library not built: {path} is missing "
                               "(run `python -m attention_forward_mode_b200.build`)")
        lib = ctypes.CDLL(path)
        vp, i64, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
        fwd_args = [vp] * 9 + [i64] * 5 + [f32, vp]
        lib.attn_jvp_fwd.argtypes = fwd_args
        lib.attn_jvp_fwd.restype = ctypes.c_int
        lib.attn_jvp_fwd_f32.argtypes = fwd_args
        lib.attn_jvp_fwd_f32.restype = ctypes.c_int
        lib.attn_jvp_fwd_f32out.argtypes = fwd_args
        lib.attn_jvp_fwd_f32out.restype = ctypes.c_int
        lib.attn_jvp_fwd_causal.argtypes = fwd_args
        lib.attn_jvp_fwd_causal.restype = ctypes.c_int
        lib.attn_jvp_fwd_f32out_causal.argtypes = fwd_args
        lib.attn_jvp_fwd_f32out_causal.restype = ctypes.c_int
        lib.attn_jvp_fwd_f32out_varlen.argtypes = [vp] * 11 + [i64] * 6 + [f32, ctypes.c_int, vp]
        lib.attn_jvp_fwd_f32out_varlen.restype = ctypes.c_int
        lib.attn_jvp_fwd_varlen.argtypes = [vp] * 11 + [i64] * 6 + [f32, ctypes.c_int, vp]
        lib.attn_jvp_fwd_varlen.restype = ctypes.c_int
        lib.attn_jvp_fwd_stats.argtypes = [vp] * 10 + [i64] * 5 + [f32, vp]
        lib.attn_jvp_fwd_stats.restype = ctypes.c_int
        lib.attn_jvp_fwd_causal_stats.argtypes = [vp] * 10 + [i64] * 5 + [f32, vp]
        lib.attn_jvp_fwd_causal_stats.restype = ctypes.c_int
        lib.attn_jvp_bwd.argtypes = [vp] * 18 + [i64] * 5 + [f32, vp, ctypes.c_uint64, vp]
        lib.attn_jvp_bwd.restype = ctypes.c_int
        lib.attn_jvp_bwd_causal.argtypes = [vp] * 18 + [i64] * 5 + [f32, vp, ctypes.c_uint64, vp]
        lib.attn_jvp_bwd_causal.restype = ctypes.c_int
        lib.attn_jvp_fwd_varlen_stats.argtypes = [vp] * 12 + [i64] * 6 + [f32, ctypes.c_int, vp]
        lib.attn_jvp_fwd_varlen_stats.restype = ctypes.c_int
        lib.attn_jvp_bwd_varlen.argtypes = ([vp] * 20 + [i64] * 7 + [f32, ctypes.c_int, vp, ctypes.c_uint64, vp])
        lib.attn_jvp_bwd_varlen.restype = ctypes.c_int
        lib.attn_jvp_bwd_step.argtypes = [ctypes.c_int] + [vp] * 18 + [i64] * 5 + [f32, vp, ctypes.c_uint64, vp]
        lib.attn_jvp_bwd_step.restype = ctypes.c_int
        lib.attn_jvp_bwd_workspace_bytes.argtypes = [i64] * 3
        lib.attn_jvp_bwd_workspace_bytes.restype = ctypes.c_uint64
        lib.attn_jvp_bwd_workspace_bytes_split.argtypes = [i64] * 4
        lib.attn_jvp_bwd_workspace_bytes_split.restype = ctypes.c_uint64
        lib.attn_jvp_bwd_key_split_parts.argtypes = [i64] * 5
        lib.attn_jvp_bwd_key_split_parts.restype = i64
        lib.attn_jvp_bwd_host.argtypes = [vp] * 18 + [i64] * 5 + [f32, vp, ctypes.c_uint64, vp]
        lib.attn_jvp_bwd_host.restype = ctypes.c_int
        lib.attn_jvp_bwd_host_workspace_bytes.argtypes = [i64] * 4
        lib.attn_jvp_bwd_host_workspace_bytes.restype = ctypes.c_uint64
        lib.attn_jvp_fwd_host.argtypes = [vp] * 9 + [i64] * 5 + [f32, vp, ctypes.c_uint64, vp]
        lib.attn_jvp_fwd_host.restype = ctypes.c_int
        lib.attn_jvp_fwd_host_noalloc.argtypes = fwd_args
        lib.attn_jvp_fwd_host_noalloc.restype = ctypes.c_int
        lib.attn_jvp_host_workspace_bytes.argtypes = [i64] * 4
        lib.attn_jvp_host_workspace_bytes.restype = ctypes.c_uint64
        lib.attn_jvp_strerror.argtypes = [ctypes.c_int]
        lib.attn_jvp_strerror.restype = ctypes.c_char_p
        lib.attn_jvp_last_cuda_error.argtypes = []
        lib.attn_jvp_last_cuda_error.restype = ctypes.c_int
        lib.attn_jvp_check_device_status.argtypes = [vp]
        lib.attn_jvp_check_device_status.restype = ctypes.c_int
        lib.attn_jvp_set_wait_bound_ns.argtypes = [ctypes.c_uint64]
        lib.attn_jvp_set_wait_bound_ns.restype = ctypes.c_int
        lib.attn_jvp_set_persistent_key_tiles.argtypes = [ctypes.c_int64]
        lib.attn_jvp_set_persistent_key_tiles.restype = ctypes.c_int
        lib.attn_jvp_set_bwd_pairs.argtypes = [ctypes.c_int]
        lib.attn_jvp_set_bwd_pairs.restype = ctypes.c_int
        lib.attn_jvp_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
        lib.attn_jvp_selftest_wait_timeout.restype = ctypes.c_int
        lib.attn_jvp_version.argtypes = []
        lib.attn_jvp_version.restype = ctypes.c_int
        _lib = lib
        return lib


def strerror(status: int) -> str:
    return load_library().attn_jvp_strerror(int(status)).decode()


def _check(status: int, where: str):
    if status != AJVP_OK:
        lib = load_library()
        msg = f"{where}: {strerror(status)} (status {status})"
        if status == AJVP_ERR_CUDA:
            msg += f", cudaError {lib.attn_jvp_last_cuda_error()}"
        raise AttnJvpError(status, msg)


def _stream_handle(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _prepare(q, k, v, tq, tk, tv, o, to, lse, dtype, want_lse, out_dtype=None):
    for name, x in (("q", q), ("k", k), ("v", v), ("tq", tq), ("tk", tk), ("tv", tv)):
        if not isinstance(x, torch.Tensor) or not x.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if x.dtype != dtype:
            raise ValueError(f"{name} must be {dtype}, got {x.dtype}")
        if x.dim() != 4 or not x.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [B, H, L, d] tensor")
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if tq.shape != q.shape:
        raise ValueError("tq must have the shape of q")
    for name, x in (("k", k), ("v", v), ("tk", tk), ("tv", tv)):
        if x.shape != (B, H, Lk, d):
            raise ValueError(f"{name} must be [B, H, Lk, d] = {(B, H, Lk, d)}, got {tuple(x.shape)}")
    out_dtype = dtype if out_dtype is None else out_dtype
    if o is None:
        o = torch.empty(q.shape, device=q.device, dtype=out_dtype)
    if to is None:
        to = torch.empty(q.shape, device=q.device, dtype=out_dtype)
    if want_lse and lse is None:
        lse = torch.empty((B, H, Lq), device=q.device, dtype=torch.float32)
    for name, x, shp, dt in (("o", o, q.shape, out_dtype), ("to", to, q.shape, out_dtype)):
        if x.shape != shp or x.dtype != dt or not x.is_contiguous() or not x.is_cuda:
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor of shape {tuple(shp)}")
    if lse is not None and (lse.shape != (B, H, Lq) or lse.dtype != torch.float32 or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous float32 [B, H, Lq] tensor")
    return o, to, lse, (B, H, Lq, Lk, d)


def attn_jvp_fwd(q, k, v, tq, tk, tv, scale=None, o=None, to=None, lse=None, stream=None, want_lse=True):
    """O, tO, lse for bf16 [B, H, L, d] CUDA tensors (d = 128), through the
    C ABI's ``attn_jvp_fwd`` (tcgen05 kernel).  Output tensors may be passed
    in; otherwise they are allocated.  Asynchronous on ``stream`` (default:
    torch's current stream)."""
    o, to, lse, (B, H, Lq, Lk, d) = _prepare(q, k, v, tq, tk, tv, o, to, lse, torch.bfloat16, want_lse)
    if scale is None:
        scale = d ** -0.5
    lib = load_library()
    rc = lib.attn_jvp_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(tq), _ptr(tk), _ptr(tv), _ptr(o), _ptr(to), _ptr(lse),
                          B, H, Lq, Lk, d, float(scale), _stream_handle(stream))
    _check(rc, "attn_jvp_fwd")
    return o, to, lse


def attn_jvp_fwd_f32out(q, k, v, tq, tk, tv, scale=None, o=None, to=None, lse=None, stream=None, want_lse=True):
    """bf16 inputs, fp32 O and tO, through ``attn_jvp_fwd_f32out`` (tcgen05
    kernel with split-bf16 probability operands; d = 128)."""
    return _fwd_f32out("attn_jvp_fwd_f32out", q, k, v, tq, tk, tv, scale, o, to, lse, stream, want_lse)


def attn_jvp_fwd_f32out_causal(q, k, v, tq, tk, tv, scale=None, o=None, to=None, lse=None, stream=None,
                               want_lse=True):
    """``attn_jvp_fwd_f32out`` with the causal mask of ``attn_jvp_fwd_causal``."""
    return _fwd_f32out("attn_jvp_fwd_f32out_causal", q, k, v, tq, tk, tv, scale, o, to, lse, stream, want_lse)


def _fwd_f32out(entry, q, k, v, tq, tk, tv, scale, o, to, lse, stream, want_lse):
    o, to, lse, (B, H, Lq, Lk, d) = _prepare(q, k, v, tq, tk, tv, o, to, lse, torch.bfloat16, want_lse,
                                            out_dtype=torch.float32)
    if scale is None:
        scale = d ** -0.5
    lib = load_library()
    rc = getattr(lib, entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(tq), _ptr(tk), _ptr(tv), _ptr(o), _ptr(to),
                             _ptr(lse), B, H, Lq, Lk, d, float(scale), _stream_handle(stream))
    _check(rc, entry)
    return o, to, lse


def attn_jvp_fwd_causal(q, k, v, tq, tk, tv, scale=None, o=None, to=None, lse=None, stream=None, want_lse=True):
    """``attn_jvp_fwd`` with a causal mask (key j visible to query row i iff
    j <= i + Lk - Lq); rows that see no key give zeros and lse = -inf."""
    o, to, lse, (B, H, Lq, Lk, d) = _prepare(q, k, v, tq, tk, tv, o, to, lse, torch.bfloat16, want_lse)
    if scale is None:
        scale = d ** -0.5
    lib = load_library()
    rc = lib.attn_jvp_fwd_causal(_ptr(q), _ptr(k), _ptr(v), _ptr(tq), _ptr(tk), _ptr(tv), _ptr(o), _ptr(to),
                                 _ptr(lse), B, H, Lq, Lk, d, float(scale), _stream_handle(stream))
    _check(rc, "attn_jvp_fwd_causal")
    return o, to, lse


def attn_jvp_fwd_varlen(q, k, v, tq, tk, tv, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, scale=None, causal=False,
                        o=None, to=None, lse=None, stream=None, want_lse=True):
    """Packed variable-length sequences: q, tq [H, total_q, d], k, v, tk, tv
    [H, total_k, d] bf16 CUDA tensors; cu_seqlens_q / _k int32 CUDA tensors of
    n_seq + 1 offsets.  Returns (o, to, lse) with o, to [H, total_q, d] and
    lse [H, total_q]."""
    o, to, lse, (H, Tq, Tk, d) = _prepare_varlen(q, k, v, tq, tk, tv, cu_seqlens_q, cu_seqlens_k, o, to, lse,
                                                 want_lse)
    if scale is None:
        scale = d ** -0.5
    lib = load_library()
    rc = lib.attn_jvp_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(tq), _ptr(tk), _ptr(tv), _ptr(o), _ptr(to),
                                 _ptr(lse), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), cu_seqlens_q.numel() - 1, H, Tq,
                                 Tk, int(max_seqlen_q), d, float(scale), int(bool(causal)), _stream_handle(stream))
    _check(rc, "attn_jvp_fwd_varlen")
    return o, to, lse


def attn_jvp_fwd_f32out_varlen(q, k, v, tq, tk, tv, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, scale=None,
                               causal=False, o=None, to=None, lse=None, stream=None, want_lse=True):
    """``attn_jvp_fwd_varlen`` with fp32 O and tO (split-bf16 probability
    operands, as ``attn_jvp_fwd_f32out``).  Returns (o, to, lse)."""
    if o is None:
        o = torch.empty(q.shape, device=q.device, dtype=torch.float32)
    if to is None:
        to = torch.empty(q.shape, device=q.device, dtype=torch.float32)
    o, to, lse, (H, Tq, Tk, d) = _prepare_varlen(q, k, v, tq, tk, tv, cu_seqlens_q, cu_seqlens_k, o, to, lse,
                                                 want_lse, out_dtype=torch.float32)
    if scale is None:
        scale = d ** -0.5
    lib = load_library()
    rc = lib.attn_jvp_fwd_f32out_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(tq), _ptr(tk), _ptr(tv), _ptr(o), _ptr(to),
                                        _ptr(lse), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), cu_seqlens_q.numel() - 1,
                                        H, Tq, Tk, int(max_seqlen_q), d, float(scale), int(bool(causal)),
                                        _stream_handle(stream))
    _check(rc, "attn_jvp_fwd_f32out_varlen")
    return o, to, lse


def attn_jvp_fwd_varlen_stats(q, k, v, tq, tk, tv, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, scale=None,
                              causal=False, o=None, to=None, lse=None, mu=None, stream=None):
    """``attn_jvp_fwd_varlen`` that also returns mu (fp32 [H, total_q]; rows
    that see no key: lse = -inf, mu = 0), for ``attn_jvp_bwd_varlen``.
    Returns (o, to, lse, mu)."""
    o, to, lse, (H, Tq, Tk, d) = _prepare_varlen(q, k, v, tq, tk, tv, cu_seqlens_q, cu_seqlens_k, o, to, lse, True)
    if mu is None:
        mu = torch.empty((H, Tq), device=q.device, dtype=torch.float32)
    if mu.shape != (H, Tq) or mu.dtype != torch.float32 or not mu.is_contiguous() or not mu.is_cuda:
        raise ValueError("mu must be a contiguous float32 CUDA [H, total_q] tensor")
    if scale is None:
        scale = d ** -0.5
    lib = load_library()
    rc = lib.attn_jvp_fwd_varlen_stats(_ptr(q), _ptr(k), _ptr(v), _ptr(tq), _ptr(tk), _ptr(tv), _ptr(o), _ptr(to),
                                       _ptr(lse), _ptr(mu), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
                                       cu_seqlens_q.numel() - 1, H, Tq, Tk, int(max_seqlen_q), d, float(scale),
                                       int(bool(causal)), _stream_handle(stream))
    _check(rc, "attn_jvp_fwd_varlen_stats")
    return o, to, lse, mu


def attn_jvp_bwd_varlen(q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, cu_seqlens_q, cu_seqlens_k,
                        max_seqlen_q, max_seqlen_k, scale=None, causal=False, grads=None, workspace=None,
                        stream=None):
    """Backward of ``attn_jvp_fwd_varlen`` through ``attn_jvp_bwd_varlen``: the
    packed tensors and offsets of the forward, o, to, lse, mu from
    ``attn_jvp_fwd_varlen_stats``, cotangents dout, dtout [H, total_q, d].
    Returns a dict dq, dk, dv, dtq, dtk, dtv (packed like q / k)."""
    _, _, _, (H, Tq, Tk, d) = _prepare_varlen(q, k, v, tq, tk, tv, cu_seqlens_q, cu_seqlens_k, o, to, lse, True)
    for name, x, shp, dt in (("mu", mu, (H, Tq), torch.float32), ("dout", dout, q.shape, torch.bfloat16),
                             ("dtout", dtout, q.shape, torch.bfloat16)):
        if not isinstance(x, torch.Tensor) or x.shape != shp or x.dtype != dt or not x.is_contiguous() \
                or not x.is_cuda:
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor of shape {tuple(shp)}")
    grads = dict(grads or {})
    for name in GRAD_NAMES:
        like = q if name in ("dq", "dtq") else k
        if grads.get(name) is None:
            grads[name] = torch.empty_like(like)
        g = grads[name]
        if g.shape != like.shape or g.dtype != torch.bfloat16 or not g.is_contiguous() or not g.is_cuda:
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape {tuple(like.shape)}")
    if scale is None:
        scale = d ** -0.5
    if workspace is None:
        workspace = torch.empty(max(1, bwd_workspace_bytes(1, H, Tq)), dtype=torch.uint8, device=q.device)
    if not workspace.is_cuda or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA uint8 tensor")
    lib = load_library()
    rc = lib.attn_jvp_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(tq), _ptr(tk), _ptr(tv), _ptr(o), _ptr(to),
                                 _ptr(lse), _ptr(mu), _ptr(dout), _ptr(dtout), *(_ptr(grads[n]) for n in GRAD_NAMES),
                                 _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), cu_seqlens_q.numel() - 1, H, Tq, Tk,
                                 int(max_seqlen_q), int(max_seqlen_k), d, float(scale), int(bool(causal)),
                                 _ptr(workspace), workspace.numel(), _stream_handle(stream))
    _check(rc, "attn_jvp_bwd_varlen")
    return grads


def _prepare_varlen(q, k, v, tq, tk, tv, cu_seqlens_q, cu_seqlens_k, o, to, lse, want_lse, out_dtype=None):
    for name, x in (("q", q), ("k", k), ("v", v), ("tq", tq), ("tk", tk), ("tv", tv)):
        if not isinstance(x, torch.Tensor) or not x.is_cuda or x.dtype != torch.bfloat16 or x.dim() != 3 \
                or not x.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA bf16 [H, total, d] tensor")
    H, Tq, d = q.shape
    Tk = k.shape[1]
    if tq.shape != q.shape or any(x.shape != (H, Tk, d) for x in (k, v, tk, tv)):
        raise ValueError("q, tq must be [H, total_q, d] and k, v, tk, tv [H, total_k, d]")
    for name, c in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if not isinstance(c, torch.Tensor) or not c.is_cuda or c.dtype != torch.int32 or c.dim() != 1 \
                or not c.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA int32 vector")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must have the same length n_seq + 1 >= 1")
    if o is None:
        o = torch.empty_like(q)
    if to is None:
        to = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((H, Tq), device=q.device, dtype=torch.float32)
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    for name, x in (("o", o), ("to", to)):
        if x.shape != q.shape or x.dtype != out_dtype or not x.is_contiguous() or not x.is_cuda:
            raise ValueError(f"{name} must be a contiguous CUDA {out_dtype} tensor of shape {tuple(q.shape)}")
    if lse is not None and (lse.shape != (H, Tq) or lse.dtype != torch.float32 or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous float32 [H, total_q] tensor")
    return o, to, lse, (H, Tq, Tk, d)


def attn_jvp_fwd_stats(q, k, v, tq, tk, tv, scale=None, o=None, to=None, lse=None, mu=None, stream=None):
    """``attn_jvp_fwd`` that also returns mu (fp32 [B, H, Lq]), the row
    statistic the backward needs beside lse.  Returns (o, to, lse, mu)."""
    return _fwd_stats("attn_jvp_fwd_stats", q, k, v, tq, tk, tv, scale, o, to, lse, mu, stream)


def attn_jvp_fwd_causal_stats(q, k, v, tq, tk, tv, scale=None, o=None, to=None, lse=None, mu=None, stream=None):
    """``attn_jvp_fwd_causal`` that also returns mu (rows that see no key:
    lse = -inf, mu = 0), for ``attn_jvp_bwd_causal``.  Returns (o, to, lse, mu)."""
    return _fwd_stats("attn_jvp_fwd_causal_stats", q, k, v, tq, tk, tv, scale, o, to, lse, mu, stream)


def _fwd_stats(entry, q, k, v, tq, tk, tv, scale, o, to, lse, mu, stream):
    o, to, lse, (B, H, Lq, Lk, d) = _prepare(q, k, v, tq, tk, tv, o, to, lse, torch.bfloat16, True)
    if mu is None:
        mu = torch.empty((B, H, Lq), device=q.device, dtype=torch.float32)
    if mu.shape != (B, H, Lq) or mu.dtype != torch.float32 or not mu.is_contiguous() or not mu.is_cuda:
        raise ValueError("mu must be a contiguous float32 CUDA [B, H, Lq] tensor")
    if scale is None:
        scale = d ** -0.5
    lib = load_library()
    rc = getattr(lib, entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(tq), _ptr(tk), _ptr(tv), _ptr(o), _ptr(to),
                             _ptr(lse), _ptr(mu), B, H, Lq, Lk, d, float(scale), _stream_handle(stream))
    _check(rc, entry)
    return o, to, lse, mu


def bwd_workspace_bytes(B: int, H: int, Lq: int, Lk: int | None = None) -> int:
    """Device workspace ``attn_jvp_bwd`` needs (row statistics); with ``Lk``,
    the size that also lets the key-side kernels split short key sequences
    (``attn_jvp_bwd_workspace_bytes_split``, for the current device)."""
    lib = load_library()
    if Lk is None:
        return int(lib.attn_jvp_bwd_workspace_bytes(int(B), int(H), int(Lq)))
    return int(lib.attn_jvp_bwd_workspace_bytes_split(int(B), int(H), int(Lq), int(Lk)))


GRAD_NAMES = ("dq", "dk", "dv", "dtq", "dtk", "dtv")


def attn_jvp_bwd(q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, scale=None, grads=None, workspace=None,
                 stream=None, step=None):
    """Gradients of <dout, O> + <dtout, tO> with respect to q, k, v, tq, tk,
    tv, through the C ABI's ``attn_jvp_bwd`` (bf16, d = 128).  o, to, lse,
    mu are the outputs of ``attn_jvp_fwd_stats`` on the same inputs.
    ``grads``: optional dict of preallocated outputs.  ``workspace``: a CUDA
    uint8 tensor (allocated per call when omitted, with room for the split
    key side: ``bwd_workspace_bytes(B, H, Lq, Lk)``; one of
    ``bwd_workspace_bytes(B, H, Lq)`` bytes runs the unsplit kernels).
    Returns a dict dq, dk, dv, dtq, dtk, dtv.  Asynchronous on ``stream``.
    ``step`` (0-3) runs one of the four steps only (``attn_jvp_bwd_step``)."""
    return _bwd("attn_jvp_bwd" if step is None else "attn_jvp_bwd_step", q, k, v, tq, tk, tv, o, to, lse, mu,
                dout, dtout, scale, grads, workspace, stream, step)


def attn_jvp_bwd_causal(q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, scale=None, grads=None, workspace=None,
                        stream=None):
    """Backward of ``attn_jvp_fwd_causal`` through ``attn_jvp_bwd_causal``;
    o, to, lse, mu from ``attn_jvp_fwd_causal_stats``.  Arguments and result
    as ``attn_jvp_bwd``."""
    return _bwd("attn_jvp_bwd_causal", q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, scale, grads, workspace,
                stream, None)


def _bwd(entry, q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, scale, grads, workspace, stream, step):
    _, _, _, (B, H, Lq, Lk, d) = _prepare(q, k, v, tq, tk, tv, o, to, lse, torch.bfloat16, True)
    for name, x, shp, dt in (("mu", mu, (B, H, Lq), torch.float32), ("dout", dout, q.shape, torch.bfloat16),
                             ("dtout", dtout, q.shape, torch.bfloat16)):
        if not isinstance(x, torch.Tensor) or x.shape != shp or x.dtype != dt or not x.is_contiguous() \
                or not x.is_cuda:
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor of shape {tuple(shp)}")
    grads = dict(grads or {})
    for name in GRAD_NAMES:
        like = q if name in ("dq", "dtq") else k
        if grads.get(name) is None:
            grads[name] = torch.empty_like(like)
        g = grads[name]
        if g.shape != like.shape or g.dtype != torch.bfloat16 or not g.is_contiguous() or not g.is_cuda:
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape {tuple(like.shape)}")
    if scale is None:
        scale = d ** -0.5
    if workspace is None:
        with torch.cuda.device(q.device):  # the split size reads this device's SM count
            nbytes = bwd_workspace_bytes(B, H, Lq, None if entry == "attn_jvp_bwd_causal" else Lk)
            workspace = torch.empty(max(1, nbytes), dtype=torch.uint8, device=q.device)
    if not workspace.is_cuda or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA uint8 tensor")
    lib = load_library()
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(tq), _ptr(tk), _ptr(tv), _ptr(o), _ptr(to), _ptr(lse), _ptr(mu),
            _ptr(dout), _ptr(dtout), *(_ptr(grads[n]) for n in GRAD_NAMES), B, H, Lq, Lk, d, float(scale),
            _ptr(workspace), workspace.numel(), _stream_handle(stream))
    if step is None:
        _check(getattr(lib, entry)(*args), entry)
    else:
        _check(lib.attn_jvp_bwd_step(int(step), *args), "attn_jvp_bwd_step")
    return grads


def bwd_key_split_parts(B: int, H: int, Lq: int, Lk: int, sm_count: int | None = None) -> int:
    """Parts into which ``attn_jvp_bwd`` (with the split workspace) cuts the
    key-side kernels' query range; ``sm_count`` defaults to the current CUDA
    device's.  Host arithmetic only."""
    if sm_count is None:
        sm_count = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    n = int(load_library().attn_jvp_bwd_key_split_parts(int(B), int(H), int(Lq), int(Lk), int(sm_count)))
    if n < 1:
        raise ValueError("invalid sizes or SM count")
    return n


def bwd_host_workspace_bytes(Lq: int, Lk: int, d: int, heads_per_chunk: int = 1) -> int:
    """Device workspace bytes for ``attn_jvp_bwd_host`` with chunks of
    ``heads_per_chunk`` (batch, head) slabs."""
    return int(load_library().attn_jvp_bwd_host_workspace_bytes(Lq, Lk, d, heads_per_chunk))


def default_bwd_heads_per_chunk(bh: int, Lq: int, Lk: int, d: int, target_bytes: int = 320 << 20) -> int:
    """Heads per staged backward chunk: about ``target_bytes`` of staged
    inputs, gradients and statistics, at least one head, at most a quarter of
    ``bh`` (so that copies overlap kernels)."""
    per_head = (8 * Lq + 8 * Lk) * d * 2 + 24 * Lq
    return max(1, min((bh + 3) // 4, target_bytes // per_head))


def attn_jvp_bwd_host(q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, scale=None, grads=None, workspace=None,
                      stream=None):
    """``attn_jvp_bwd`` on HOST tensors (pinned for overlap): the library
    stages head chunks through a device workspace and overlaps the copies with
    the kernels.  Inputs as ``attn_jvp_bwd`` but in host memory; ``grads``: an
    optional dict of preallocated host outputs.  ``workspace`` is a CUDA uint8
    tensor (allocated for ``default_bwd_heads_per_chunk`` heads when
    omitted).  Asynchronous on ``stream``; synchronise it before reading the
    gradients.  Returns a dict dq, dk, dv, dtq, dtk, dtv."""
    for name, x in (("q", q), ("k", k), ("v", v), ("tq", tq), ("tk", tk), ("tv", tv)):
        if not isinstance(x, torch.Tensor) or x.is_cuda or x.dtype != torch.bfloat16 or x.dim() != 4 \
                or not x.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 [B, H, L, d] host tensor")
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if tq.shape != q.shape or any(x.shape != (B, H, Lk, d) for x in (k, v, tk, tv)):
        raise ValueError("q, tq must be [B, H, Lq, d] and k, v, tk, tv [B, H, Lk, d]")
    for name, x, shp, dt in (("o", o, q.shape, torch.bfloat16), ("to", to, q.shape, torch.bfloat16),
                             ("dout", dout, q.shape, torch.bfloat16), ("dtout", dtout, q.shape, torch.bfloat16),
                             ("lse", lse, (B, H, Lq), torch.float32), ("mu", mu, (B, H, Lq), torch.float32)):
        if not isinstance(x, torch.Tensor) or x.is_cuda or x.shape != shp or x.dtype != dt or not x.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {dt} host tensor of shape {tuple(shp)}")
    pin = q.is_pinned()
    grads = dict(grads or {})
    for name in GRAD_NAMES:
        like = q if name in ("dq", "dtq") else k
        if grads.get(name) is None:
            grads[name] = torch.empty(like.shape, dtype=torch.bfloat16, pin_memory=pin)
        g = grads[name]
        if g.is_cuda or g.shape != like.shape or g.dtype != torch.bfloat16 or not g.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 host tensor of shape {tuple(like.shape)}")
    if scale is None:
        scale = d ** -0.5
    if workspace is None:
        nh = default_bwd_heads_per_chunk(B * H, Lq, Lk, d)
        workspace = torch.empty(max(1, bwd_host_workspace_bytes(Lq, Lk, d, nh)), dtype=torch.uint8, device="cuda")
    if not workspace.is_cuda or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA uint8 tensor")
    lib = load_library()
    rc = lib.attn_jvp_bwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(tq), _ptr(tk), _ptr(tv), _ptr(o), _ptr(to), _ptr(lse),
                               _ptr(mu), _ptr(dout), _ptr(dtout), *(_ptr(grads[n]) for n in GRAD_NAMES), B, H, Lq, Lk,
                               d, float(scale), _ptr(workspace), workspace.numel(), _stream_handle(stream))
    _check(rc, "attn_jvp_bwd_host")
    return grads


def attn_jvp_fwd_f32(q, k, v, tq, tk, tv, scale=None, o=None, to=None, lse=None, stream=None, want_lse=True):
    """fp32-I/O variant through ``attn_jvp_fwd_f32`` (CUDA-core kernel, d <= 256)."""
    o, to, lse, (B, H, Lq, Lk, d) = _prepare(q, k, v, tq, tk, tv, o, to, lse, torch.float32, want_lse)
    if scale is None:
        scale = d ** -0.5
    lib = load_library()
    rc = lib.attn_jvp_fwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(tq), _ptr(tk), _ptr(tv), _ptr(o), _ptr(to),
                              _ptr(lse), B, H, Lq, Lk, d, float(scale), _stream_handle(stream))
    _check(rc, "attn_jvp_fwd_f32")
    return o, to, lse


def host_workspace_bytes(Lq: int, Lk: int, d: int, heads_per_chunk: int = 1) -> int:
    """Device workspace ``attn_jvp_fwd_host`` needs for chunks of ``heads_per_chunk`` heads."""
    return int(load_library().attn_jvp_host_workspace_bytes(int(Lq), int(Lk), int(d), int(heads_per_chunk)))


def _prepare_host(q, k, v, tq, tk, tv, o, to, lse, want_lse):
    for name, x in (("q", q), ("k", k), ("v", v), ("tq", tq), ("tk", tk), ("tv", tv)):
        if not isinstance(x, torch.Tensor) or x.is_cuda or x.dtype != torch.bfloat16 or x.dim() != 4 \
                or not x.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 [B, H, L, d] host tensor")
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if tq.shape != q.shape or any(x.shape != (B, H, Lk, d) for x in (k, v, tk, tv)):
        raise ValueError("q, tq must be [B, H, Lq, d] and k, v, tk, tv [B, H, Lk, d]")
    pin = q.is_pinned()
    if o is None:
        o = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=pin)
    if to is None:
        to = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=pin)
    if want_lse and lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, pin_memory=pin)
    for name, x in (("o", o), ("to", to)):
        if x.is_cuda or x.shape != q.shape or x.dtype != torch.bfloat16 or not x.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 host tensor of shape {tuple(q.shape)}")
    if lse is not None and (lse.is_cuda or lse.shape != (B, H, Lq) or lse.dtype != torch.float32
                            or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous float32 [B, H, Lq] host tensor")
    return o, to, lse, (B, H, Lq, Lk, d)


def default_heads_per_chunk(bh: int, Lq: int, Lk: int, d: int, target_bytes: int = 64 << 20) -> int:
    """Heads per staged chunk: about ``target_bytes`` of inputs and outputs
    (enough to keep each copy long against its launch cost), at least one
    head, at most a quarter of ``bh`` (so that copies overlap kernels)."""
    per_head = (4 * Lq + 4 * Lk) * d * 2 + 4 * Lq
    return max(1, min((bh + 3) // 4, target_bytes // per_head))


def attn_jvp_fwd_host(q, k, v, tq, tk, tv, scale=None, o=None, to=None, lse=None, workspace=None,
                      stream=None, want_lse=True):
    """``attn_jvp_fwd`` on bf16 [B, H, L, d] HOST tensors (pinned for overlap):
    the library stages head chunks through a device workspace, overlapping
    the copies in and out with the kernel.  ``workspace`` is a CUDA uint8
    tensor (allocated for ``default_heads_per_chunk`` heads when omitted).  The
    call is asynchronous on ``stream``; synchronise it before reading o, to,
    lse."""
    o, to, lse, (B, H, Lq, Lk, d) = _prepare_host(q, k, v, tq, tk, tv, o, to, lse, want_lse)
    if scale is None:
        scale = d ** -0.5
    if workspace is None:
        workspace = torch.empty(max(1, host_workspace_bytes(Lq, Lk, d, default_heads_per_chunk(B * H, Lq, Lk, d))),
                                dtype=torch.uint8, device="cuda")
    if not workspace.is_cuda or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA uint8 tensor")
    lib = load_library()
    rc = lib.attn_jvp_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(tq), _ptr(tk), _ptr(tv), _ptr(o), _ptr(to),
                               _ptr(lse), B, H, Lq, Lk, d, float(scale), _ptr(workspace), workspace.numel(),
                               _stream_handle(stream))
    _check(rc, "attn_jvp_fwd_host")
    return o, to, lse


def attn_jvp_fwd_host_noalloc(q, k, v, tq, tk, tv, scale=None, o=None, to=None, lse=None, stream=None,
                              want_lse=True):
    """``attn_jvp_fwd_host`` staged through the library's static 64 MiB device
    scratch instead of a workspace (the C call allocates no device memory).
    Calls on different streams must not overlap.  Asynchronous on ``stream``."""
    o, to, lse, (B, H, Lq, Lk, d) = _prepare_host(q, k, v, tq, tk, tv, o, to, lse, want_lse)
    if scale is None:
        scale = d ** -0.5
    lib = load_library()
    rc = lib.attn_jvp_fwd_host_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(tq), _ptr(tk), _ptr(tv), _ptr(o), _ptr(to),
                                       _ptr(lse), B, H, Lq, Lk, d, float(scale), _stream_handle(stream))
    _check(rc, "attn_jvp_fwd_host_noalloc")
    return o, to, lse


def attn_jvp(q, k, v, tq, tk, tv, scale=None, **kw):
    """Dispatch on the input dtype: bf16 -> attn_jvp_fwd, fp32 -> attn_jvp_fwd_f32."""
    if q.dtype == torch.bfloat16:
        return attn_jvp_fwd(q, k, v, tq, tk, tv, scale, **kw)
    if q.dtype == torch.float32:
        return attn_jvp_fwd_f32(q, k, v, tq, tk, tv, scale, **kw)
    raise ValueError(f"unsupported dtype {q.dtype}")


def check_device_status(stream=None) -> int:
    """Synchronise ``stream`` and read-and-clear the device status word."""
    return load_library().attn_jvp_check_device_status(_stream_handle(stream))


def set_wait_bound_ns(ns: int) -> None:
    _check(load_library().attn_jvp_set_wait_bound_ns(int(ns)), "attn_jvp_set_wait_bound_ns")


DEFAULT_PERSISTENT_KEY_TILES = 32


def set_persistent_key_tiles(max_key_tiles: int) -> None:
    """Key sequences of at most ``max_key_tiles`` 64-key tiles use the
    persistent form of the unmasked bf16 forward (0: never).  Process-wide."""
    _check(load_library().attn_jvp_set_persistent_key_tiles(int(max_key_tiles)),
           "attn_jvp_set_persistent_key_tiles")


DEFAULT_BWD_PAIRS = False


def set_bwd_pairs(on: bool) -> None:
    """The backward's unmasked dQ/dtQ and dK/dtK kernels as CTA pairs sharing
    each tensor-core product, or one CTA per row tile (the default,
    ``DEFAULT_BWD_PAIRS``).  Process-wide."""
    _check(load_library().attn_jvp_set_bwd_pairs(1 if on else 0), "attn_jvp_set_bwd_pairs")


def selftest_wait_timeout(bound_ns: int, stream=None) -> None:
    _check(load_library().attn_jvp_selftest_wait_timeout(int(bound_ns), _stream_handle(stream)),
           "attn_jvp_selftest_wait_timeout")


def version() -> int:
    return load_library().attn_jvp_version()
