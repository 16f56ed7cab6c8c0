"""attn_jvp_autograd: gradients through torch autograd of a loss built from O
and tO equal the direct attn_jvp_bwd (attn_jvp_bwd_causal) call bit for bit,
and the fp64 oracle within the backward bound; an output left out of the loss
gets a zero cotangent."""
import pytest
import torch

import attention_forward_mode_b200 as ajvp
import oracle
from attention_forward_mode_b200.workloads import custom, make_cotangents
from gpu_common import gpu_inputs, max_rel

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "tq", "tk", "tv")


def test_autograd_matches_direct_backward():
    w = custom(2, 2, 260, 300, 128)
    inp = gpu_inputs(w, seed=31)
    cot = make_cotangents(w, seed=32, device="cuda")
    leaves = {n: inp[n].clone().requires_grad_(True) for n in NAMES}
    o, to = ajvp.attn_jvp_autograd(*(leaves[n] for n in NAMES), w.scale)
    loss = (o.float() * cot["dout"].float()).sum() + (to.float() * cot["dtout"].float()).sum()
    loss.backward()
    ro, rto, rlse, rmu = ajvp.attn_jvp_fwd_stats(*(inp[n] for n in NAMES), w.scale)
    g = ajvp.attn_jvp_bwd(*(inp[n] for n in NAMES), ro, rto, rlse, rmu, cot["dout"], cot["dtout"], w.scale)
    torch.cuda.synchronize()
    for n, gn in zip(NAMES, ("dq", "dk", "dv", "dtq", "dtk", "dtv")):
        assert torch.equal(leaves[n].grad, g[gn]), n
    ref = oracle.attn_jvp_bwd(*(inp[n] for n in NAMES), cot["dout"], cot["dtout"], w.scale)
    for n, gn in zip(NAMES, ("dq", "dk", "dv", "dtq", "dtk", "dtv")):
        assert max_rel(leaves[n].grad.float().cpu().numpy(), ref[gn]) <= 2e-2, n


def test_loss_on_the_tangent_only():
    w = custom(1, 2, 200, 150, 128)
    inp = gpu_inputs(w, seed=33)
    cot = make_cotangents(w, seed=34, device="cuda")
    leaves = {n: inp[n].clone().requires_grad_(True) for n in NAMES}
    _, to = ajvp.attn_jvp_autograd(*(leaves[n] for n in NAMES), w.scale)
    (to.float() * cot["dtout"].float()).sum().backward()
    zero = torch.zeros_like(cot["dout"])
    ref = oracle.attn_jvp_bwd(*(inp[n] for n in NAMES), zero, cot["dtout"], w.scale)
    for n, gn in zip(NAMES, ("dq", "dk", "dv", "dtq", "dtk", "dtv")):
        assert max_rel(leaves[n].grad.float().cpu().numpy(), ref[gn]) <= 2e-2, n


def test_causal_autograd_matches_direct_backward():
    w = custom(1, 2, 300, 240, 128)  # Lq > Lk: the first 60 rows see no key
    inp = gpu_inputs(w, seed=35)
    cot = make_cotangents(w, seed=36, device="cuda")
    leaves = {n: inp[n].clone().requires_grad_(True) for n in NAMES}
    o, to = ajvp.attn_jvp_autograd(*(leaves[n] for n in NAMES), w.scale, causal=True)
    loss = (o.float() * cot["dout"].float()).sum() + (to.float() * cot["dtout"].float()).sum()
    loss.backward()
    ro, rto, rlse, rmu = ajvp.attn_jvp_fwd_causal_stats(*(inp[n] for n in NAMES), w.scale)
    g = ajvp.attn_jvp_bwd_causal(*(inp[n] for n in NAMES), ro, rto, rlse, rmu, cot["dout"], cot["dtout"], w.scale)
    torch.cuda.synchronize()
    for n, gn in zip(NAMES, ("dq", "dk", "dv", "dtq", "dtk", "dtv")):
        assert torch.equal(leaves[n].grad, g[gn]), n
    ref = oracle.attn_jvp_bwd_causal(*(inp[n] for n in NAMES), cot["dout"], cot["dtout"], w.scale)
    for n, gn in zip(NAMES, ("dq", "dk", "dv", "dtq", "dtk", "dtv")):
        assert max_rel(leaves[n].grad.float().cpu().numpy(), ref[gn]) <= 2e-2, n
