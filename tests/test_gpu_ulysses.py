"""The Ulysses wrapper on the GPU through NCCL: with a one-rank NCCL group the
two all-to-all exchanges run for real (as identity exchanges) around the CUDA
kernel, and the result must equal a direct attn_jvp_fwd call bit for bit; the
same for the training path (forward keeping its head shards, backward
exchanges around attn_jvp_bwd), unmasked and causal.
(Exchanges across several ranks are checked on CPU over gloo.)"""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist

import attention_forward_mode_b200 as ajvp
from attention_forward_mode_b200.ulysses import ulysses_attn_jvp
from attention_forward_mode_b200.workloads import custom, make_inputs

pytestmark = pytest.mark.gpu


def test_one_rank_nccl_equals_direct_call():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        w = custom(1, 4, 384, 640, 128)
        inp = make_inputs(w, seed=3, device="cuda")
        a = ulysses_attn_jvp(inp["q"], inp["k"], inp["v"], inp["tq"], inp["tk"], inp["tv"], scale=w.scale)
        b = ajvp.attn_jvp_fwd(inp["q"], inp["k"], inp["v"], inp["tq"], inp["tk"], inp["tv"], w.scale)
        torch.cuda.synchronize()
        for x, y in zip(a, b):
            assert torch.equal(x, y)
        # training path: forward keeping its head shards, then the backward exchanges
        from attention_forward_mode_b200.ulysses import ulysses_attn_jvp_bwd, ulysses_attn_jvp_train
        from attention_forward_mode_b200.workloads import make_cotangents
        names = ("q", "k", "v", "tq", "tk", "tv")
        cot = make_cotangents(w, seed=4, device="cuda")
        o, to, lse, ctx = ulysses_attn_jvp_train(*(inp[n] for n in names), scale=w.scale)
        g = ulysses_attn_jvp_bwd(ctx, cot["dout"], cot["dtout"])
        ro, rto, rlse, rmu = ajvp.attn_jvp_fwd_stats(*(inp[n] for n in names), w.scale)
        rg = ajvp.attn_jvp_bwd(*(inp[n] for n in names), ro, rto, rlse, rmu, cot["dout"], cot["dtout"], w.scale)
        torch.cuda.synchronize()
        assert torch.equal(o, ro) and torch.equal(to, rto) and torch.equal(lse, rlse)
        for n in ajvp.GRAD_NAMES:
            assert torch.equal(g[n], rg[n]), n
        # the causal training path: the default local steps are the causal kernels
        o, to, lse, ctx = ulysses_attn_jvp_train(*(inp[n] for n in names), scale=w.scale, causal=True)
        g = ulysses_attn_jvp_bwd(ctx, cot["dout"], cot["dtout"])
        ro, rto, rlse, rmu = ajvp.attn_jvp_fwd_causal_stats(*(inp[n] for n in names), w.scale)
        rg = ajvp.attn_jvp_bwd_causal(*(inp[n] for n in names), ro, rto, rlse, rmu, cot["dout"], cot["dtout"],
                                      w.scale)
        torch.cuda.synchronize()
        assert torch.equal(o, ro) and torch.equal(to, rto) and torch.equal(lse, rlse)
        for n in ajvp.GRAD_NAMES:
            assert torch.equal(g[n], rg[n]), n
    finally:
        dist.destroy_process_group()
