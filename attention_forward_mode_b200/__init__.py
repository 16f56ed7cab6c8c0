"""Fused attention + Jacobian-vector product (forward-mode tangent) for
NVIDIA B200 (sm_100a): O = softmax(s Q K^T) V and tO, its derivative along
(tQ, tK, tV), in one tiled pass -- the attention hot path of rCM's
continuous-time consistency distillation.

The computation lives in the CUDA library ``libattnjvp.so`` (C ABI in
``include/attn_jvp.h``); this package is its ctypes binding plus the seeded
synthetic-input generator.  The library is loaded on first use and a missing
build raises.
"""
from ._binding import (  # noqa: F401
    AJVP_ERR_CUDA,
    AJVP_ERR_INVALID_ARG,
    AJVP_ERR_MISALIGNED,
    AJVP_ERR_TIMEOUT,
    AJVP_ERR_TOO_LARGE,
    AJVP_ERR_UNSUPPORTED_DEVICE,
    AJVP_ERR_UNSUPPORTED_DIM,
    AJVP_ERR_WORKSPACE,
    AJVP_OK,
    DEFAULT_BWD_PAIRS,
    DEFAULT_PERSISTENT_KEY_TILES,
    GRAD_NAMES,
    AttnJvpError,
    attn_jvp,
    attn_jvp_bwd,
    attn_jvp_bwd_causal,
    attn_jvp_bwd_varlen,
    attn_jvp_bwd_host,
    attn_jvp_fwd,
    attn_jvp_fwd_causal,
    attn_jvp_fwd_f32,
    attn_jvp_fwd_f32out,
    attn_jvp_fwd_f32out_causal,
    attn_jvp_fwd_f32out_varlen,
    attn_jvp_fwd_host,
    attn_jvp_fwd_host_noalloc,
    attn_jvp_fwd_stats,
    attn_jvp_fwd_causal_stats,
    attn_jvp_fwd_varlen,
    attn_jvp_fwd_varlen_stats,
    bwd_host_workspace_bytes,
    bwd_key_split_parts,
    bwd_workspace_bytes,
    check_device_status,
    default_bwd_heads_per_chunk,
    default_heads_per_chunk,
    host_workspace_bytes,
    load_library,
    selftest_wait_timeout,
    set_bwd_pairs,
    set_persistent_key_tiles,
    set_wait_bound_ns,
    strerror,
    version,
)

from .autograd import AttnJvpFunction, attn_jvp_autograd  # noqa: E402,F401

__all__ = [
    "AttnJvpFunction", "attn_jvp_autograd", "attn_jvp", "attn_jvp_bwd", "attn_jvp_bwd_causal",
    "attn_jvp_fwd_causal_stats", "attn_jvp_bwd_varlen", "attn_jvp_fwd_varlen_stats", "attn_jvp_bwd_host",
    "bwd_host_workspace_bytes", "default_bwd_heads_per_chunk", "attn_jvp_fwd_causal", "attn_jvp_fwd_varlen",
    "attn_jvp_fwd_stats", "bwd_workspace_bytes", "bwd_key_split_parts", "attn_jvp_fwd", "attn_jvp_fwd_f32",
    "attn_jvp_fwd_f32out", "attn_jvp_fwd_f32out_causal", "attn_jvp_fwd_f32out_varlen", "attn_jvp_fwd_host",
    "attn_jvp_fwd_host_noalloc", "check_device_status", "default_heads_per_chunk", "host_workspace_bytes",
    "load_library", "selftest_wait_timeout", "set_bwd_pairs", "set_persistent_key_tiles", "DEFAULT_BWD_PAIRS",
    "DEFAULT_PERSISTENT_KEY_TILES",
    "set_wait_bound_ns", "strerror", "version", "AttnJvpError",
]
