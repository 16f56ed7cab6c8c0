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


@pytest.mark.parametrize("Lq,Lk", [(300, 260),     # one CTA per query tile
                                   (19000, 300)])  # 298 query tiles: the persistent forward
def test_forward_and_backward_in_a_graph(Lq, Lk):
    w = custom(1, 2, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=1)
    cot = make_cotangents(w, seed=2, device="cuda")
    o, to, lse, mu = (torch.empty_like(inp["q"]), torch.empty_like(inp["q"]),
                      torch.empty((1, 2, Lq), device="cuda"), torch.empty((1, 2, Lq), device="cuda"))
    grads = {n: torch.empty_like(inp["q"] if n in ("dq", "dtq") else inp["k"]) for n in ajvp.GRAD_NAMES}
    ws = torch.empty(ajvp.bwd_workspace_bytes(1, 2, Lq), dtype=torch.uint8, device="cuda")

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
