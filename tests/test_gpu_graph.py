"""The device-buffer entry points allocate nothing and never synchronise, so a
caller can capture them into a CUDA graph (after a first eager call on the
device, which does the one-time set-up).  Replays must equal eager calls
bit for bit, including after the inputs change in place."""
import pytest
import torch

import attention_forward_mode_b200 as ajvp
from attention_forward_mode_b200.workloads import custom, make_cotangents
from gpu_common import gpu_inputs

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "tq", "tk", "tv")


@pytest.mark.parametrize("Lq,Lk,split", [(300, 260, False),     # one CTA per query tile
                                         (19000, 300, False),   # 298 query tiles: the persistent forward
                                         (3000, 300, True)])    # the key side split over the queries
def test_forward_and_backward_in_a_graph(Lq, Lk, split):
    w = custom(1, 2, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=1)
    cot = make_cotangents(w, seed=2, device="cuda")
    o, to, lse, mu = (torch.empty_like(inp["q"]), torch.empty_like(inp["q"]),
                      torch.empty((1, 2, Lq), device="cuda"), torch.empty((1, 2, Lq), device="cuda"))
    grads = {n: torch.empty_like(inp["q"] if n in ("dq", "dtq") else inp["k"]) for n in ajvp.GRAD_NAMES}
    ws = torch.empty(ajvp.bwd_workspace_bytes(1, 2, Lq, Lk if split else None), dtype=torch.uint8, device="cuda")

    def step(stream=None):
        ajvp.attn_jvp_fwd_stats(*(inp[n] for n in NAMES), w.scale, o=o, to=to, lse=lse, mu=mu, stream=stream)
        ajvp.attn_jvp_bwd(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], w.scale,
                          grads=grads, workspace=ws, stream=stream)

    step()  # one-time set-up on the device, outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step(stream=s)
    for seed in (3, 4):
        new = gpu_inputs(w, seed=seed)
        for n in NAMES:
            inp[n].copy_(new[n])
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (o, to, lse, mu)] + [grads[n].clone() for n in ajvp.GRAD_NAMES]
        step()
        torch.cuda.synchronize()
        ref = [o, to, lse, mu] + [grads[n] for n in ajvp.GRAD_NAMES]
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
    assert ajvp.check_device_status() == ajvp.AJVP_OK


@pytest.mark.parametrize("mode", ["causal", "varlen"])
def test_masked_forward_and_backward_in_a_graph(mode):
    # the causal pair on dense tensors, the packed pair on three sequences (one
    # without keys), captured after one eager call and replayed on changed inputs
    if mode == "causal":
        w = custom(1, 2, 300, 260, 128)
        inp = gpu_inputs(w, seed=5)
        cot = make_cotangents(w, seed=6, device="cuda")
        shp_q, shp_s = inp["q"].shape, (1, 2, 300)
    else:
        lq, lk = [150, 90, 40], [130, 0, 220]
        gen = torch.Generator().manual_seed(5)
        inp = {n: torch.randn((2, sum(lq) if n in ("q", "tq") else sum(lk), 128),
                              generator=gen).to(torch.bfloat16).cuda() for n in NAMES}
        cot = {n: torch.randn((2, sum(lq), 128), generator=gen).to(torch.bfloat16).cuda()
               for n in ("dout", "dtout")}
        cq = torch.tensor([0, 150, 240, 280], dtype=torch.int32, device="cuda")
        ck = torch.tensor([0, 130, 130, 350], dtype=torch.int32, device="cuda")
        shp_q, shp_s = inp["q"].shape, (2, sum(lq))
    o, to = torch.empty(shp_q, dtype=torch.bfloat16, device="cuda"), torch.empty(shp_q, dtype=torch.bfloat16,
                                                                                   device="cuda")
    lse, mu = torch.empty(shp_s, device="cuda"), torch.empty(shp_s, device="cuda")
    grads = {n: torch.empty_like(inp["q"] if n in ("dq", "dtq") else inp["k"]) for n in ajvp.GRAD_NAMES}
    ws = torch.empty(ajvp.bwd_workspace_bytes(1, shp_s[-2] if mode == "varlen" else 2, shp_s[-1]),
                     dtype=torch.uint8, device="cuda")
    s = 128 ** -0.5

    def step(stream=None):
        if mode == "causal":
            ajvp.attn_jvp_fwd_causal_stats(*(inp[n] for n in NAMES), s, o=o, to=to, lse=lse, mu=mu, stream=stream)
            ajvp.attn_jvp_bwd_causal(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], s,
                                     grads=grads, workspace=ws, stream=stream)
        else:
            ajvp.attn_jvp_fwd_varlen_stats(*(inp[n] for n in NAMES), cq, ck, 150, s, o=o, to=to, lse=lse, mu=mu,
                                           stream=stream)
            ajvp.attn_jvp_bwd_varlen(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], cq, ck,
                                     150, 220, s, grads=grads, workspace=ws, stream=stream)

    step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st):
            step(stream=st)
    for seed in (7, 8):
        gen2 = torch.Generator().manual_seed(seed)
        for n in NAMES:
            inp[n].copy_(torch.randn(inp[n].shape, generator=gen2).to(torch.bfloat16).cuda())
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (o, to, lse, mu)] + [grads[n].clone() for n in ajvp.GRAD_NAMES]
        step()
        torch.cuda.synchronize()
        ref = [o, to, lse, mu] + [grads[n] for n in ajvp.GRAD_NAMES]
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
    assert ajvp.check_device_status() == ajvp.AJVP_OK
