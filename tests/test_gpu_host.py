"""attn_jvp_fwd_host (host buffers, head chunks staged through a device
workspace with copies overlapped with the kernel) against attn_jvp_fwd on the
same inputs: each chunk is the same kernel on the same slabs, so the outputs
must be bit-identical; plus the workspace rules."""
import pytest
import torch

import attention_forward_mode_b200 as ajvp
from attention_forward_mode_b200.workloads import custom
from gpu_common import gpu_inputs

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "tq", "tk", "tv")


def device_ref(inp, scale):
    o, to, lse = ajvp.attn_jvp_fwd(*(inp[n] for n in NAMES), scale)
    torch.cuda.synchronize()
    return o.cpu(), to.cpu(), lse.cpu()


def host_run(inp, scale, pinned=True, heads_per_chunk=None, want_lse=True):
    h = {n: (t.cpu().pin_memory() if pinned else t.cpu()) for n, t in inp.items()}
    ws = None
    if heads_per_chunk is not None:
        B, H, Lq, d = h["q"].shape
        ws = torch.empty(ajvp.host_workspace_bytes(Lq, h["k"].shape[2], d, heads_per_chunk), dtype=torch.uint8,
                         device="cuda")
    out = ajvp.attn_jvp_fwd_host(*(h[n] for n in NAMES), scale, workspace=ws, want_lse=want_lse)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("B,H,Lq,Lk,chunk", [(1, 1, 1, 1, None),        # one head, one chunk
                                             (2, 3, 300, 700, None),    # 6 heads in chunks of 2
                                             (1, 7, 129, 257, 2),       # ragged last chunk
                                             (1, 5, 640, 512, 1),       # one head per chunk
                                             (2, 2, 200, 64, 4),        # all heads in one chunk
                                             (1, 3, 20000, 512, 1)])    # persistent kernel per chunk
def test_host_equals_device(B, H, Lq, Lk, chunk):
    w = custom(B, H, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=B * 100 + H * 10 + Lq)
    ref = device_ref(inp, w.scale)
    got = host_run(inp, w.scale, heads_per_chunk=chunk)
    for name, a, b in zip(("o", "to", "lse"), got, ref):
        assert not a.is_cuda
        assert torch.equal(a, b), name


def test_pageable_host_memory_and_no_lse():
    w = custom(1, 4, 256, 384, 128)
    inp = gpu_inputs(w, seed=3)
    ref = device_ref(inp, w.scale)
    o, to, lse = host_run(inp, w.scale, pinned=False, heads_per_chunk=1, want_lse=False)
    assert lse is None
    assert torch.equal(o, ref[0]) and torch.equal(to, ref[1])


def test_two_calls_reuse_workspace():
    w = custom(1, 6, 200, 300, 128)
    a, b = gpu_inputs(w, seed=4), gpu_inputs(w, seed=5)
    ws = torch.empty(ajvp.host_workspace_bytes(w.Lq, w.Lk, w.d, 2), dtype=torch.uint8, device="cuda")
    ha = {n: t.cpu().pin_memory() for n, t in a.items()}
    hb = {n: t.cpu().pin_memory() for n, t in b.items()}
    ra = ajvp.attn_jvp_fwd_host(*(ha[n] for n in NAMES), w.scale, workspace=ws)
    rb = ajvp.attn_jvp_fwd_host(*(hb[n] for n in NAMES), w.scale, workspace=ws)
    torch.cuda.synchronize()
    for got, inp in ((ra, a), (rb, b)):
        ref = device_ref(inp, w.scale)
        assert all(torch.equal(x, y) for x, y in zip(got, ref))


def test_workspace_too_small_is_rejected():
    w = custom(1, 2, 128, 128, 128)
    inp = {n: t.cpu() for n, t in gpu_inputs(w, seed=6).items()}
    need = ajvp.host_workspace_bytes(w.Lq, w.Lk, w.d, 1)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ajvp.AttnJvpError) as ei:
        ajvp.attn_jvp_fwd_host(*(inp[n] for n in NAMES), w.scale, workspace=ws)
    assert ei.value.status == ajvp.AJVP_ERR_WORKSPACE


def _bwd_case(w, seed):
    from attention_forward_mode_b200.workloads import make_cotangents
    inp = gpu_inputs(w, seed=seed)
    cot = make_cotangents(w, seed=seed + 1, device="cuda")
    o, to, lse, mu = ajvp.attn_jvp_fwd_stats(*(inp[n] for n in NAMES), w.scale)
    # the staged path's workspace holds each chunk's row statistics only, so its key
    # side never splits: compare with a device call whose workspace is as small
    ws = torch.empty(ajvp.bwd_workspace_bytes(w.B, w.H, w.Lq), dtype=torch.uint8, device="cuda")
    ref = ajvp.attn_jvp_bwd(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], w.scale,
                            workspace=ws)
    torch.cuda.synchronize()
    dev = {**inp, "o": o, "to": to, "lse": lse, "mu": mu, **cot}
    return dev, {n: g.cpu() for n, g in ref.items()}


def _bwd_host(dev, scale, pinned=True, workspace=None):
    h = {n: (t.cpu().pin_memory() if pinned else t.cpu()) for n, t in dev.items()}
    got = ajvp.attn_jvp_bwd_host(*(h[n] for n in NAMES), h["o"], h["to"], h["lse"], h["mu"], h["dout"], h["dtout"],
                                 scale, workspace=workspace)
    torch.cuda.synchronize()
    return got


@pytest.mark.parametrize("B,H,Lq,Lk,chunk", [(1, 1, 64, 64, None),       # one head, one chunk
                                             (2, 3, 300, 700, 2),        # 6 heads in chunks of 2
                                             (1, 7, 129, 257, 2),        # ragged last chunk
                                             (1, 5, 640, 512, 1),        # one head per chunk
                                             (2, 2, 200, 64, 4)])        # all heads in one chunk
def test_bwd_host_equals_device(B, H, Lq, Lk, chunk):
    """attn_jvp_bwd_host runs the same kernels on each chunk's slabs: the
    gradients equal attn_jvp_bwd's bit for bit."""
    w = custom(B, H, Lq, Lk, 128)
    dev, ref = _bwd_case(w, seed=B * 100 + H * 10 + Lq)
    ws = None
    if chunk is not None:
        ws = torch.empty(ajvp.bwd_host_workspace_bytes(Lq, Lk, 128, chunk), dtype=torch.uint8, device="cuda")
    got = _bwd_host(dev, w.scale, workspace=ws)
    for n in ajvp.GRAD_NAMES:
        assert not got[n].is_cuda
        assert torch.equal(got[n], ref[n]), n


def test_bwd_host_pageable_memory_and_small_workspace_rejected():
    w = custom(1, 3, 200, 260, 128)
    dev, ref = _bwd_case(w, seed=21)
    got = _bwd_host(dev, w.scale, pinned=False)
    for n in ajvp.GRAD_NAMES:
        assert torch.equal(got[n], ref[n]), n
    small = torch.empty(ajvp.bwd_host_workspace_bytes(200, 260, 128, 1) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ajvp.AttnJvpError):
        _bwd_host(dev, w.scale, workspace=small)


def test_bwd_host_without_query_rows_zeroes_key_gradients():
    w = custom(1, 2, 0, 96, 128)
    h = {n: torch.zeros((1, 2, 0 if n in ("q", "tq", "o", "to", "dout", "dtout") else 96, 128), dtype=torch.bfloat16)
         for n in ("q", "k", "v", "tq", "tk", "tv", "o", "to", "dout", "dtout")}
    h["lse"] = torch.zeros((1, 2, 0), dtype=torch.float32)
    h["mu"] = torch.zeros((1, 2, 0), dtype=torch.float32)
    grads = {n: torch.full((1, 2, 0 if n in ("dq", "dtq") else 96, 128), 7.0, dtype=torch.bfloat16)
             for n in ajvp.GRAD_NAMES}
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    out = ajvp.attn_jvp_bwd_host(*(h[n] for n in NAMES), h["o"], h["to"], h["lse"], h["mu"], h["dout"], h["dtout"],
                                 w.scale, grads=grads, workspace=ws)
    torch.cuda.synchronize()
    for n in ("dk", "dv", "dtk", "dtv"):
        assert torch.count_nonzero(out[n]) == 0, n
