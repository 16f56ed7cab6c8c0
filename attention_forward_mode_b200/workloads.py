"""Seeded synthetic inputs for the attention-JVP path.

This module only draws random numbers; it holds none of the attention or JVP
arithmetic, so both the CUDA path's tests and the fp64 oracle can take their
inputs from it.

The shapes stand in for the attention layers of the diffusion transformers rCM
distils (anthology record LIT-783, results summary for Tables 1-3: Cosmos-
Predict2 image models, Wan2.1 480p video with text conditioning): an image
token grid of 64x64, video latent grids of 21x30x52 and 21x45x80 tokens, and
512 text tokens for cross-attention.  No dataset or trained weights are used.

Draw order, fixed so a seed names one input set: from one CPU
torch.Generator seeded with ``seed``, standard-normal fp32 draws for
Q, K, V, tQ, tK, tV in that order, each [B, H, L, d]; then, for the
cross-attention workload only, per-key factors uK and uV ~ U(0.5, 2) of shape
[B, H, Lk] (uniform draw * 1.5 + 0.5).  Each tensor is multiplied by its
stated standard deviation (and K, V rows by uK, uV), then rounded to the I/O
dtype (round-to-nearest-even), all on the host; only the rounded tensor is
moved to the target device.  So one seed names the same tensors whatever the
device, and a host can re-draw exactly what a GPU run used.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Lq: int
    Lk: int
    d: int
    dtype: str  # "bf16" or "f32": I/O element type; accumulation is fp32
    scale: float
    q_std: float = 1.0
    k_std: float = 1.0
    v_std: float = 1.0
    t_std: float = 1.0
    kv_row_scale: bool = False  # per-key U(0.5, 2) factors on K and V rows
    note: str = ""

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def flops(self) -> int:
        """12 * Lq * Lk * d per head: six Lq x Lk x d products."""
        return 12 * self.B * self.H * self.Lq * self.Lk * self.d

    @property
    def elem_size(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    @property
    def io_bytes(self) -> int:
        """Compulsory HBM bytes: Q, tQ, O, tO once; K, tK, V, tV once; lse."""
        e = self.elem_size
        bh = self.B * self.H
        return bh * (4 * self.Lq * self.d * e + 4 * self.Lk * self.d * e + 4 * self.Lq)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("selfattn_f32_b1h2_l128_d64", 1, 2, 128, 128, 64, "f32", 1.0 / 8.0,
                 note="small fp32-I/O self-attention, all tensors N(0,1)"),
        Workload("image_selfattn_b2h12_l4096_d128", 2, 12, 4096, 4096, 128, "bf16",
                 1.0 / math.sqrt(128.0), t_std=0.1,
                 note="image DiT token grid 64x64; tangents N(0, 0.1^2)"),
        Workload("video_selfattn_b1h12_l32760_d128", 1, 12, 32760, 32760, 128, "bf16",
                 1.0 / math.sqrt(128.0),
                 note="video latent grid 21x30x52 flattened; all N(0,1)"),
        Workload("video_crossattn_b1h40_lq32760_lk512_d128", 1, 40, 32760, 512, 128, "bf16",
                 1.0 / math.sqrt(128.0), kv_row_scale=True,
                 note="video tokens attending 512 text tokens; K, V rows scaled by U(0.5,2)"),
        Workload("video_selfattn_large_b1h40_l75600_d128", 1, 40, 75600, 75600, 128, "bf16",
                 1.0 / math.sqrt(128.0), q_std=2.0, k_std=2.0,
                 note="video latent grid 21x45x80 flattened; Q, K ~ N(0, 2^2) for peaky rows"),
    ]
}

# The order the workloads are listed in (small fp32 case first).
WORKLOAD_ORDER = list(WORKLOADS)
BENCH_WORKLOAD = "video_selfattn_b1h12_l32760_d128"


def custom(B, H, Lq, Lk, d, dtype="bf16", scale=None, **kw) -> Workload:
    """An ad-hoc workload (edge-case tests): N(0,1) everywhere unless overridden."""
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    name = f"custom_b{B}h{H}_lq{Lq}_lk{Lk}_d{d}_{dtype}"
    return Workload(name, B, H, Lq, Lk, d, dtype, float(scale), **kw)


def make_inputs(w: Workload | str, seed: int = 0, device="cpu", dtype=None):
    """Q, K, V, tQ, tK, tV as a dict of contiguous [B, H, L, d] tensors on
    `device`, drawn and rounded on the host (the same tensors for every
    device)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    out_dtype = dtype if dtype is not None else w.torch_dtype
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shapes = {"q": (w.B, w.H, w.Lq, w.d), "k": (w.B, w.H, w.Lk, w.d),
              "v": (w.B, w.H, w.Lk, w.d), "tq": (w.B, w.H, w.Lq, w.d),
              "tk": (w.B, w.H, w.Lk, w.d), "tv": (w.B, w.H, w.Lk, w.d)}
    std = {"q": w.q_std, "k": w.k_std, "v": w.v_std, "tq": w.t_std, "tk": w.t_std, "tv": w.t_std}

    def finish(name, x):
        if std[name] != 1.0:
            x.mul_(std[name])
        return x.to(out_dtype).contiguous().to(device)

    out, raw = {}, {}
    for name in ("q", "k", "v", "tq", "tk", "tv"):
        x = torch.randn(shapes[name], generator=g, dtype=torch.float32)
        if w.kv_row_scale and name in ("k", "v"):
            raw[name] = x  # the per-key factors are drawn after all six tensors
        else:
            out[name] = finish(name, x)
        del x
    if w.kv_row_scale:
        uk = torch.rand((w.B, w.H, w.Lk), generator=g, dtype=torch.float32) * 1.5 + 0.5
        uv = torch.rand((w.B, w.H, w.Lk), generator=g, dtype=torch.float32) * 1.5 + 0.5
        out["k"] = finish("k", raw.pop("k").mul_(uk[..., None]))
        out["v"] = finish("v", raw.pop("v").mul_(uv[..., None]))
    return {n: out[n] for n in ("q", "k", "v", "tq", "tk", "tv")}


def make_cotangents(w: Workload | str, seed: int = 1, device="cpu", dtype=None):
    """Cotangents dO, dtO of the outputs (for the backward pass): standard
    normal [B, H, Lq, d] tensors, drawn in that order from their own seeded
    CPU generator and rounded on the host (the pages give no training signal
    to imitate)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    out_dtype = dtype if dtype is not None else w.torch_dtype
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shape = (w.B, w.H, w.Lq, w.d)
    return {n: torch.randn(shape, generator=g, dtype=torch.float32).to(out_dtype).contiguous().to(device)
            for n in ("dout", "dtout")}


def sample_rows(Lq: int, n: int, seed: int = 0, tile: int = 128):
    """A seeded subset of query rows that always contains the first and last
    rows, both sides of every 128-row tile boundary it can reach and the
    ragged tail, topped up with uniformly drawn rows."""
    must = {0, Lq - 1}
    for b in (tile - 1, tile, 2 * tile - 1, 2 * tile):
        if b < Lq:
            must.add(b)
    tail0 = (Lq // tile) * tile
    if tail0 < Lq:
        must.add(tail0)
        if tail0 > 0:
            must.add(tail0 - 1)
    g = torch.Generator().manual_seed(seed)
    extra = torch.randperm(Lq, generator=g)[: max(0, n - len(must))].tolist()
    return sorted(must.union(extra))[: max(n, len(must))]
