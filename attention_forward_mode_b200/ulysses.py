"""Ulysses context parallelism for the attention + JVP forward pass.

rCM (anthology record LIT-783, §3.2 / App. C) runs its FlashAttention-2 JVP
kernel under Ulysses context parallelism, with the tangents distributed like
Q, K and V.  Each rank holds a sequence shard of every head:

    q, tq        [B, H, Lq / P, d]      k, v, tk, tv  [B, H, Lk / P, d]

An all-to-all turns that into full sequences for H / P heads per rank, the
local fused kernel runs on them, and a second all-to-all returns O, tO and
lse to sequence shards:

    o, to        [B, H, Lq / P, d]      lse           [B, H, Lq / P]

Rank r's sequence shard is rows r*L/P .. (r+1)*L/P - 1; rank r computes
heads r*H/P .. (r+1)*H/P - 1.  H, Lq and Lk must divide by P.  The Q-side
tensors (q, tq) and the K-side tensors (k, v, tk, tv) each travel in one
packed all-to-all, the outputs in one more (plus one for lse).  The exchange
uses torch.distributed (NCCL on GPUs); the attention itself is the library's
kernel (``local_fn``, by default the C ABI entry point for the inputs'
dtype).

``ulysses_attn_jvp_train`` / ``ulysses_attn_jvp_bwd`` add the backward: the
forward keeps its head-sharded inputs and outputs, the backward sends the
cotangents dO, dtO to head shards, runs the local backward there and returns
the six gradients to sequence shards.

``causal=True`` selects the causal kernels as the local step: after the
exchange every rank holds whole sequences in their original order, so the
mask (key j visible to query i iff j <= i + Lk - Lq) applies unchanged.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from ._binding import attn_jvp


def _to_heads(x: torch.Tensor, world: int, group) -> torch.Tensor:
    """[n, B, H, Ls, d] sequence shard -> [n, B, H/P, P*Ls, d] head shard."""
    n, B, H, Ls, d = x.shape
    hp = H // world
    # [n, B, P, H/P, Ls, d] -> [P, n, B, H/P, Ls, d]: chunk p goes to rank p
    send = x.reshape(n, B, world, hp, Ls, d).permute(2, 0, 1, 3, 4, 5).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[p] = rank p's sequence rows for my heads -> [n, B, H/P, P, Ls, d]
    return recv.permute(1, 2, 3, 0, 4, 5).reshape(n, B, hp, world * Ls, d)


def _to_sequence(y: torch.Tensor, world: int, group) -> torch.Tensor:
    """[n, B, H/P, P*Ls, e] head shard -> [n, B, H, Ls, e] sequence shard."""
    n, B, hp, L, e = y.shape
    Ls = L // world
    # [n, B, H/P, P, Ls, e] -> [P, n, B, H/P, Ls, e]: sequence chunk p goes to rank p
    send = y.reshape(n, B, hp, world, Ls, e).permute(3, 0, 1, 2, 4, 5).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[p] = my sequence rows of rank p's heads -> [n, B, P, H/P, Ls, e]
    return recv.permute(1, 2, 0, 3, 4, 5).reshape(n, B, world * hp, Ls, e)


def ulysses_attn_jvp(q, k, v, tq, tk, tv, scale=None, group=None, local_fn=None, causal=False):
    """O, tO, lse for sequence-sharded inputs (see the module docstring).

    ``local_fn(q, k, v, tq, tk, tv, scale) -> (o, to, lse)`` computes the
    attention JVP of the gathered head shard; it defaults to the CUDA kernel
    (``attn_jvp``, or ``attn_jvp_fwd_causal`` with ``causal``).  Collective
    calls are made in the same order on every rank.
    """
    grouped = dist.is_initialized()
    world = dist.get_world_size(group) if grouped else 1
    B, H, Lqs, d = q.shape
    Lks = k.shape[2]
    if H % world != 0:
        raise ValueError(f"heads ({H}) must divide by the group size ({world})")
    if scale is None:
        scale = d ** -0.5
    if local_fn is not None:
        fn = local_fn
    elif causal:
        from ._binding import attn_jvp_fwd_causal
        fn = attn_jvp_fwd_causal
    else:
        fn = attn_jvp
    if not grouped:  # no process group: the plain local call
        return fn(q, k, v, tq, tk, tv, scale)

    qs = _to_heads(torch.stack((q, tq)), world, group)        # [2, B, H/P, Lq, d]
    ks = _to_heads(torch.stack((k, v, tk, tv)), world, group)  # [4, B, H/P, Lk, d]
    o, to, lse = fn(qs[0].contiguous(), ks[0].contiguous(), ks[1].contiguous(), qs[1].contiguous(),
                    ks[2].contiguous(), ks[3].contiguous(), scale)
    out = _to_sequence(torch.stack((o, to)), world, group)      # [2, B, H, Lq/P, d]
    lse_s = _to_sequence(lse.unsqueeze(0).unsqueeze(-1).contiguous(), world, group)[0, ..., 0]
    assert out.shape[3] == Lqs and ks.shape[3] == Lks * world
    return out[0], out[1], lse_s


def ulysses_attn_jvp_train(q, k, v, tq, tk, tv, scale=None, group=None, local_fwd=None, causal=False):
    """Forward of ``ulysses_attn_jvp`` that also keeps what the backward needs.

    Returns (o, to, lse, ctx): the sequence-sharded outputs as
    ``ulysses_attn_jvp`` gives them, and ``ctx`` for ``ulysses_attn_jvp_bwd``
    holding the head-sharded inputs and the forward's head-sharded O, tO, lse
    and mu.  ``local_fwd(q, k, v, tq, tk, tv, scale) -> (o, to, lse, mu)``
    defaults to the library's ``attn_jvp_fwd_stats`` (``attn_jvp_fwd_causal_stats``
    with ``causal``, which ``ulysses_attn_jvp_bwd`` then follows).
    """
    from ._binding import attn_jvp_fwd_causal_stats, attn_jvp_fwd_stats
    grouped = dist.is_initialized()
    world = dist.get_world_size(group) if grouped else 1
    B, H, Lqs, d = q.shape
    if H % world != 0:
        raise ValueError(f"heads ({H}) must divide by the group size ({world})")
    if scale is None:
        scale = d ** -0.5
    fn = local_fwd if local_fwd is not None else (attn_jvp_fwd_causal_stats if causal else attn_jvp_fwd_stats)
    if not grouped:
        o, to, lse, mu = fn(q, k, v, tq, tk, tv, scale)
        ctx = dict(inputs=(q, k, v, tq, tk, tv), outputs=(o, to, lse, mu), scale=scale, world=1, causal=causal)
        return o, to, lse, ctx
    qs = _to_heads(torch.stack((q, tq)), world, group)        # [2, B, H/P, Lq, d]
    ks = _to_heads(torch.stack((k, v, tk, tv)), world, group)  # [4, B, H/P, Lk, d]
    inputs = (qs[0].contiguous(), ks[0].contiguous(), ks[1].contiguous(), qs[1].contiguous(), ks[2].contiguous(),
              ks[3].contiguous())
    o, to, lse, mu = fn(*inputs, scale)
    out = _to_sequence(torch.stack((o, to)), world, group)
    lse_s = _to_sequence(lse.unsqueeze(0).unsqueeze(-1).contiguous(), world, group)[0, ..., 0]
    ctx = dict(inputs=inputs, outputs=(o, to, lse, mu), scale=scale, world=world, causal=causal)
    return out[0], out[1], lse_s, ctx


def ulysses_attn_jvp_bwd(ctx, dout, dtout, group=None, local_bwd=None):
    """Backward of ``ulysses_attn_jvp_train``: the gradients of
    <dout, O> + <dtout, tO> with respect to the six sequence-sharded inputs.

    ``dout``, ``dtout``: sequence-sharded cotangents [B, H, Lq/P, d].  They go
    to head shards (one packed all-to-all), the local backward runs on the
    head-sharded tensors the forward kept, and the gradients return to
    sequence shards (one all-to-all for the query side, one for the key
    side).  ``local_bwd(q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout,
    scale) -> dict`` defaults to the library's ``attn_jvp_bwd`` (or
    ``attn_jvp_bwd_causal`` when the forward was causal).  Returns a dict dq,
    dk, dv, dtq, dtk, dtv shaped like the inputs.
    """
    from ._binding import attn_jvp_bwd, attn_jvp_bwd_causal
    fn = local_bwd if local_bwd is not None else (attn_jvp_bwd_causal if ctx.get("causal") else attn_jvp_bwd)
    world = ctx["world"]
    if world == 1:
        return fn(*ctx["inputs"], *ctx["outputs"], dout, dtout, ctx["scale"])
    cot = _to_heads(torch.stack((dout, dtout)), world, group)  # [2, B, H/P, Lq, d]
    g = fn(*ctx["inputs"], *ctx["outputs"], cot[0].contiguous(), cot[1].contiguous(), ctx["scale"])
    qside = _to_sequence(torch.stack((g["dq"], g["dtq"])), world, group)
    kside = _to_sequence(torch.stack((g["dk"], g["dv"], g["dtk"], g["dtv"])), world, group)
    return {"dq": qside[0], "dtq": qside[1], "dk": kside[0], "dv": kside[1], "dtk": kside[2], "dtv": kside[3]}
