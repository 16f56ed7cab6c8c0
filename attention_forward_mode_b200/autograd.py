"""PyTorch autograd for the fused attention + JVP: a differentiable
``(o, to) = attn_jvp_autograd(q, k, v, tq, tk, tv)`` whose forward is the C
ABI's ``attn_jvp_fwd_stats`` and whose backward is ``attn_jvp_bwd`` (with
``causal=True``: ``attn_jvp_fwd_causal_stats`` and ``attn_jvp_bwd_causal``), so that
a loss built from both O and its tangent tO (as rCM's consistency-distillation
objective is) back-propagates into Q, K, V and the tangents through the
library's kernels only.  Plumbing: argument marshalling and saved tensors;
every step of the computation runs in the CUDA library.
"""
from __future__ import annotations

import torch

from ._binding import attn_jvp_bwd, attn_jvp_bwd_causal, attn_jvp_fwd_causal_stats, attn_jvp_fwd_stats

__all__ = ["AttnJvpFunction", "attn_jvp_autograd"]


class AttnJvpFunction(torch.autograd.Function):
    """Forward: O and tO (bf16, [B, H, Lq, d]); backward: the six gradients."""

    @staticmethod
    def forward(ctx, q, k, v, tq, tk, tv, scale, causal=False):
        q, k, v, tq, tk, tv = (x.contiguous() for x in (q, k, v, tq, tk, tv))
        fwd = attn_jvp_fwd_causal_stats if causal else attn_jvp_fwd_stats
        o, to, lse, mu = fwd(q, k, v, tq, tk, tv, scale)
        ctx.save_for_backward(q, k, v, tq, tk, tv, o, to, lse, mu)
        ctx.scale = scale
        ctx.causal = causal
        return o, to

    @staticmethod
    def backward(ctx, dout, dtout):
        q, k, v, tq, tk, tv, o, to, lse, mu = ctx.saved_tensors
        # an output that does not reach the loss has no cotangent: zeros
        dout = torch.zeros_like(o) if dout is None else dout.to(o.dtype).contiguous()
        dtout = torch.zeros_like(to) if dtout is None else dtout.to(to.dtype).contiguous()
        bwd = attn_jvp_bwd_causal if ctx.causal else attn_jvp_bwd
        g = bwd(q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, ctx.scale)
        return g["dq"], g["dk"], g["dv"], g["dtq"], g["dtk"], g["dtv"], None, None


def attn_jvp_autograd(q, k, v, tq, tk, tv, scale=None, causal=False):
    """Differentiable (O, tO) for bf16 [B, H, L, 128] CUDA tensors; ``causal``:
    key j visible to query row i iff j <= i + (Lk - Lq)."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    return AttnJvpFunction.apply(q, k, v, tq, tk, tv, float(scale), bool(causal))
