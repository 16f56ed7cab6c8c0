"""attn_jvp_bwd (gradients of <dO, O> + <dtO, tO> with respect to Q, K, V and
the tangents) against the fp64 backward oracle on the same bf16 inputs.

Bound on max|err| / max|ref| per gradient: 2e-2, the bound the forward
holds its tangent output to.  The kernel rounds the per-score gradient
factors (S_bar, dS_bar, P, P.*(u-mu)) to bf16 before the tensor-core
products (relative 2^-9 each, accumulated in fp32 with random signs) and
rounds the gradients to bf16 (2^-9); it also uses the forward's bf16 O and
tO in the row statistics a and D, whose rounding (2^-9 of |dO||O|) enters
S_bar through the difference P_bar - D."""
import numpy as np
import pytest
import torch

import attention_forward_mode_b200 as ajvp
import oracle
from attention_forward_mode_b200.workloads import WORKLOADS, custom, make_cotangents, sample_rows
from gpu_common import gpu_inputs, max_rel

pytestmark = pytest.mark.gpu

TOL = 2e-2
NAMES = ("q", "k", "v", "tq", "tk", "tv")


def run(inp, cot, scale):
    o, to, lse, mu = ajvp.attn_jvp_fwd_stats(*(inp[n] for n in NAMES), scale)
    g = ajvp.attn_jvp_bwd(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], scale)
    torch.cuda.synchronize()
    assert ajvp.check_device_status() == ajvp.AJVP_OK
    return g, (o, to, lse, mu)


@pytest.mark.parametrize("B,H,Lq,Lk", [(1, 1, 1, 1), (1, 2, 64, 64), (1, 2, 129, 127), (2, 3, 300, 700),
                                       (1, 1, 257, 1000), (1, 2, 1000, 130)])
def test_shapes_full(B, H, Lq, Lk):
    w = custom(B, H, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=Lq + 7 * Lk)
    cot = make_cotangents(w, seed=Lq + Lk, device="cuda")
    got, _ = run(inp, cot, w.scale)
    ref = oracle.attn_jvp_bwd(*(inp[n] for n in NAMES), cot["dout"], cot["dtout"], w.scale)
    err = {n: max_rel(got[n].float().cpu().numpy(), ref[n]) for n in ("dq", "dk", "dv", "dtq", "dtk", "dtv")}
    print(w.name, err)
    for n, e in err.items():
        assert e <= TOL, f"{w.name}: {n} max-rel error {e:.3e} > {TOL} ({err})"


def test_mu_output():
    w = custom(2, 2, 200, 333, 128)
    inp = gpu_inputs(w, seed=3)
    o, to, lse, mu = ajvp.attn_jvp_fwd_stats(*(inp[n] for n in NAMES), w.scale)
    o2, to2, lse2 = ajvp.attn_jvp_fwd(*(inp[n] for n in NAMES), w.scale)
    torch.cuda.synchronize()
    # the statistics variant is the same kernel: identical outputs
    assert torch.equal(o, o2) and torch.equal(to, to2) and torch.equal(lse, lse2)
    x = {n: inp[n].double().cpu() for n in NAMES}
    s = w.scale
    p = torch.softmax(s * x["q"] @ x["k"].mT, dim=-1)
    ds = s * (x["tq"] @ x["k"].mT + x["q"] @ x["tk"].mT)
    ref = (p * ds).sum(-1)
    err = (mu.double().cpu() - ref).abs().max().item() / ds.abs().max().item()
    assert err < 1e-3, err


def test_zero_cotangents_give_zero_gradients():
    w = custom(1, 2, 150, 200, 128)
    inp = gpu_inputs(w, seed=4)
    cot = {n: torch.zeros((w.B, w.H, w.Lq, w.d), dtype=torch.bfloat16, device="cuda") for n in ("dout", "dtout")}
    got, _ = run(inp, cot, w.scale)
    for n, g in got.items():
        assert torch.count_nonzero(g).item() == 0, n


def test_zero_tangent_cotangent_gives_zero_tangent_gradients():
    # dtO = 0: the tangent inputs do not affect L, so dtq, dtk, dtv are exactly 0
    w = custom(1, 2, 190, 260, 128)
    inp = gpu_inputs(w, seed=5)
    cot = make_cotangents(w, seed=6, device="cuda")
    cot["dtout"].zero_()
    got, _ = run(inp, cot, w.scale)
    for n in ("dtq", "dtk", "dtv"):
        assert torch.count_nonzero(got[n]).item() == 0, n
    ref = oracle.attn_jvp_bwd(*(inp[n] for n in NAMES), cot["dout"], cot["dtout"], w.scale)
    for n in ("dq", "dk", "dv"):
        assert max_rel(got[n].float().cpu().numpy(), ref[n]) <= TOL, n


def test_deterministic():
    w = custom(1, 3, 333, 444, 128)
    inp = gpu_inputs(w, seed=8)
    cot = make_cotangents(w, seed=9, device="cuda")
    a, _ = run(inp, cot, w.scale)
    b, _ = run(inp, cot, w.scale)
    for n in a:
        assert torch.equal(a[n], b[n]), n


def test_workspace_too_small():
    w = custom(1, 1, 64, 64, 128)
    inp = gpu_inputs(w, seed=10)
    cot = make_cotangents(w, seed=11, device="cuda")
    o, to, lse, mu = ajvp.attn_jvp_fwd_stats(*(inp[n] for n in NAMES), w.scale)
    ws = torch.empty(ajvp.bwd_workspace_bytes(1, 1, 64) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ajvp.AttnJvpError) as ei:
        ajvp.attn_jvp_bwd(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], w.scale,
                          workspace=ws)
    assert ei.value.status == ajvp.AJVP_ERR_WORKSPACE


def test_image_workload_sampled():
    w = WORKLOADS["image_selfattn_b2h12_l4096_d128"]
    inp = gpu_inputs(w)
    cot = make_cotangents(w, device="cuda")
    got, _ = run(inp, cot, w.scale)
    h = 5  # one (batch, head); the oracle's key-side sums need every query row
    rows = sample_rows(w.Lq, 24)
    keys = sample_rows(w.Lk, 24, seed=1)
    fl = {n: t.reshape(-1, t.shape[-2], t.shape[-1])[h] for n, t in {**inp, **cot}.items()}
    ref = oracle.attn_jvp_bwd(*(fl[n][None] for n in NAMES), fl["dout"][None], fl["dtout"][None], w.scale,
                              qrows=rows, krows=keys)
    err = {}
    for n in ("dq", "dtq"):
        err[n] = max_rel(got[n].reshape(-1, w.Lq, w.d)[h][rows].float().cpu().numpy(), ref[n][0])
    for n in ("dk", "dv", "dtk", "dtv"):
        err[n] = max_rel(got[n].reshape(-1, w.Lk, w.d)[h][keys].float().cpu().numpy(), ref[n][0])
    print(w.name, err)
    for n, e in err.items():
        assert e <= TOL, f"{n}: {e:.3e} ({err})"


def test_steps_equal_all_in_one():
    w = custom(2, 2, 300, 270, 128)
    inp = gpu_inputs(w, seed=12)
    cot = make_cotangents(w, seed=13, device="cuda")
    full, (o, to, lse, mu) = run(inp, cot, w.scale)
    # the whole call's default workspace (the split size): the steps take the same split
    ws = torch.empty(ajvp.bwd_workspace_bytes(w.B, w.H, w.Lq, w.Lk), dtype=torch.uint8, device="cuda")
    grads = None
    for step in (0, 3, 1, 2):  # steps 1-3 only need step 0 before them
        grads = ajvp.attn_jvp_bwd(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], w.scale,
                                  grads=grads, workspace=ws, step=step)
    torch.cuda.synchronize()
    for n in full:
        assert torch.equal(full[n], grads[n]), n


def test_video_workload_query_side_sampled():
    # the bench's backward configuration (B=1, H=12, L=32760): dQ and dtQ rows can be
    # computed by the oracle one by one (each needs all keys of its head, no other rows)
    w = WORKLOADS["video_selfattn_b1h12_l32760_d128"]
    inp = gpu_inputs(w)
    cot = make_cotangents(w, device="cuda")
    got, _ = run(inp, cot, w.scale)
    rows = sample_rows(w.Lq, 12)
    err = {"dq": 0.0, "dtq": 0.0}
    for h in (0, 7, w.B * w.H - 1):
        fl = {n: t.reshape(-1, t.shape[-2], t.shape[-1])[h] for n, t in {**inp, **cot}.items()}
        ref = oracle.attn_jvp_bwd(*(fl[n][None] for n in NAMES), fl["dout"][None], fl["dtout"][None], w.scale,
                                  qrows=rows, krows=[])
        for n in ("dq", "dtq"):
            e = max_rel(got[n].reshape(-1, w.Lq, w.d)[h][rows].float().cpu().numpy(), ref[n][0])
            err[n] = max(err[n], e)
    print(w.name, err)
    for n, e in err.items():
        assert e <= TOL, f"{n}: {e:.3e}"
    del inp, cot, got
    torch.cuda.empty_cache()


def test_video_workload_key_side_sampled():
    # the same configuration's key-side kernels (dK+dtK, dV+dtV): the oracle's gradient
    # of a key needs every query row of its head, so one head and 8 keys, including
    # both sides of the first row-tile boundaries and the ragged last tile
    w = WORKLOADS["video_selfattn_b1h12_l32760_d128"]
    inp = gpu_inputs(w)
    cot = make_cotangents(w, device="cuda")
    got, _ = run(inp, cot, w.scale)
    h = 5
    keys = sample_rows(w.Lk, 8, seed=1)
    fl = {n: t.reshape(-1, t.shape[-2], t.shape[-1])[h].cpu() for n, t in {**inp, **cot}.items()}
    ref = oracle.attn_jvp_bwd(*(fl[n][None] for n in NAMES), fl["dout"][None], fl["dtout"][None], w.scale,
                              qrows=[], krows=keys)
    err = {n: max_rel(got[n].reshape(-1, w.Lk, w.d)[h][keys].float().cpu().numpy(), ref[n][0])
           for n in ("dk", "dv", "dtk", "dtv")}
    print(w.name, keys, err)
    for n, e in err.items():
        assert e <= TOL, f"{n}: {e:.3e}"
    del inp, cot, got
    torch.cuda.empty_cache()
