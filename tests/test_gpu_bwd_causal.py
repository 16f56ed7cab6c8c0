"""attn_jvp_bwd_causal (the backward of the causal forward) against the fp64
masked backward oracle on the same bf16 inputs.

Key j is visible to query row i iff j <= i + (Lk - Lq) (bottom-right
aligned).  Bound on max|err| / max|ref| per gradient: 2e-2, as for the
unmasked backward (the same bf16 roundings of the per-score factors and of
the gradients; hidden pairs contribute exact zeros)."""
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
GRADS = ("dq", "dk", "dv", "dtq", "dtk", "dtv")


def run(inp, cot, scale):
    o, to, lse, mu = ajvp.attn_jvp_fwd_causal_stats(*(inp[n] for n in NAMES), scale)
    g = ajvp.attn_jvp_bwd_causal(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], scale)
    torch.cuda.synchronize()
    assert ajvp.check_device_status() == ajvp.AJVP_OK
    return g, (o, to, lse, mu)


@pytest.mark.parametrize("B,H,Lq,Lk", [(1, 1, 1, 1), (1, 2, 64, 64), (1, 2, 200, 200), (1, 2, 129, 127),
                                       (2, 3, 300, 700), (1, 1, 257, 1000), (1, 2, 1000, 130), (1, 2, 300, 100)])
def test_shapes_full(B, H, Lq, Lk):
    w = custom(B, H, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=3 * Lq + Lk)
    cot = make_cotangents(w, seed=Lq + 5 * Lk, device="cuda")
    got, _ = run(inp, cot, w.scale)
    ref = oracle.attn_jvp_bwd_causal(*(inp[n] for n in NAMES), cot["dout"], cot["dtout"], w.scale)
    err = {n: max_rel(got[n].float().cpu().numpy(), ref[n]) for n in GRADS}
    print(w.name, err)
    for n, e in err.items():
        assert e <= TOL, f"{w.name}: {n} max-rel error {e:.3e} > {TOL} ({err})"
    if Lq > Lk:  # rows 0 .. Lq-Lk-1 see no key: their gradients are exact zeros
        for n in ("dq", "dtq"):
            assert torch.count_nonzero(got[n][:, :, :Lq - Lk]).item() == 0, n


def test_causal_stats_forward():
    w = custom(1, 2, 300, 200, 128)  # Lq > Lk: the first 100 rows see no key
    inp = gpu_inputs(w, seed=21)
    o, to, lse, mu = ajvp.attn_jvp_fwd_causal_stats(*(inp[n] for n in NAMES), w.scale)
    o2, to2, lse2 = ajvp.attn_jvp_fwd_causal(*(inp[n] for n in NAMES), w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(to, to2) and torch.equal(lse, lse2)
    x = {n: inp[n].double().cpu() for n in NAMES}
    s = w.scale
    i = torch.arange(w.Lq)[:, None]
    j = torch.arange(w.Lk)[None, :]
    hidden = j > i + (w.Lk - w.Lq)
    sc = (s * x["q"] @ x["k"].mT).masked_fill(hidden, float("-inf"))
    empty = hidden.all(-1)
    p = torch.softmax(sc, dim=-1).nan_to_num(0.0)
    ds = s * (x["tq"] @ x["k"].mT + x["q"] @ x["tk"].mT)
    ref = (p * ds).sum(-1)
    err = (mu.double().cpu() - ref).abs().max().item() / ds.abs().max().item()
    assert err < 1e-3, err
    assert torch.all(mu[:, :, empty] == 0) and torch.all(torch.isneginf(lse[:, :, empty]))


def test_single_query_row_equals_unmasked():
    # one query row sees every key (bottom-right alignment): the causal kernels do
    # the unmasked arithmetic, bit for bit (the unmasked call with its dQ / dK
    # kernels one CTA per row tile, as the causal ones run: the CTA-pair form adds
    # each tile's products in another order)
    w = custom(1, 3, 1, 517, 128)
    inp = gpu_inputs(w, seed=22)
    cot = make_cotangents(w, seed=23, device="cuda")
    got, _ = run(inp, cot, w.scale)
    o, to, lse, mu = ajvp.attn_jvp_fwd_stats(*(inp[n] for n in NAMES), w.scale)
    ajvp.set_bwd_pairs(False)
    try:
        ref = ajvp.attn_jvp_bwd(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], w.scale)
        torch.cuda.synchronize()
    finally:
        ajvp.set_bwd_pairs(ajvp.DEFAULT_BWD_PAIRS)
    for n in GRADS:
        assert torch.equal(got[n], ref[n]), n


def test_zero_cotangents_and_determinism():
    w = custom(1, 2, 333, 280, 128)
    inp = gpu_inputs(w, seed=24)
    cot = make_cotangents(w, seed=25, device="cuda")
    a, _ = run(inp, cot, w.scale)
    b, _ = run(inp, cot, w.scale)
    for n in a:
        assert torch.equal(a[n], b[n]), n
    zero = {n: torch.zeros_like(cot[n]) for n in cot}
    z, _ = run(inp, zero, w.scale)
    for n, g in z.items():
        assert torch.count_nonzero(g).item() == 0, n


def test_video_workload_sampled():
    # the video self-attention configuration (B=1, H=12, L=32760) with the causal mask:
    # dQ, dtQ rows one by one (each needs only its own visible keys) on three heads, and
    # the key-side gradients of 8 keys of one head (each needs every query row).
    # Row 0 sees one key: there O = V_0 and tO = tV_0 exactly, so the exact dq_0 and
    # dtq_0 are 0, while the kernel's row statistic D_0 = <dO, O> + <dtO, tO> - a mu is
    # formed from the forward's bf16 outputs (as FlashAttention forms D from its bf16
    # O); their deviation dD_0 enters S_bar undiluted by P, giving
    # |dq_0| <= s |dD_0| max|K_0| (a_0 is exact, O_0 = bf16(V_0) = V_0).  That row is
    # held to this bound; the others to the relative bound.
    w = WORKLOADS["video_selfattn_b1h12_l32760_d128"]
    inp = gpu_inputs(w)
    cot = make_cotangents(w, device="cuda")
    got, (o, to, _, _) = run(inp, cot, w.scale)
    rows = sample_rows(w.Lq, 12)
    assert rows[0] == 0
    err = {n: 0.0 for n in GRADS}
    for h in (0, 7, w.B * w.H - 1):
        fl = {n: t.reshape(-1, t.shape[-2], t.shape[-1])[h].cpu() for n, t in {**inp, **cot}.items()}
        ref = oracle.attn_jvp_bwd_causal(*(fl[n][None] for n in NAMES), fl["dout"][None], fl["dtout"][None],
                                         w.scale, qrows=rows, krows=[])
        for n in ("dq", "dtq"):
            g = got[n].reshape(-1, w.Lq, w.d)[h][rows].float().cpu().numpy()
            e = max_rel(g[1:], ref[n][0][1:])
            err[n] = max(err[n], e)
        f64 = lambda t: t.double().cpu().numpy()  # noqa: E731
        o0 = f64(o.reshape(-1, w.Lq, w.d)[h][0])
        to0 = f64(to.reshape(-1, w.Lq, w.d)[h][0])
        dD = float(f64(fl["dout"][0]) @ (o0 - f64(fl["v"][0])) + f64(fl["dtout"][0]) @ (to0 - f64(fl["tv"][0])))
        bound = w.scale * abs(dD) * float(np.abs(f64(fl["k"][0])).max()) * 1.01
        scale_ref = float(np.abs(ref["dq"][0]).max())
        dq0 = float(np.abs(got["dq"].reshape(-1, w.Lq, w.d)[h][0].float().cpu().numpy()).max())
        dtq0 = float(np.abs(got["dtq"].reshape(-1, w.Lq, w.d)[h][0].float().cpu().numpy()).max())
        print(f"head {h} row 0: |dq_0| {dq0:.3e} (bound {bound:.3e}), |dtq_0| {dtq0:.3e}")
        assert dq0 <= bound + 1e-3 * scale_ref, (h, dq0, bound)
        assert dtq0 <= 1e-3 * scale_ref, (h, dtq0)
    h = 5
    keys = sample_rows(w.Lk, 8, seed=1)
    fl = {n: t.reshape(-1, t.shape[-2], t.shape[-1])[h].cpu() for n, t in {**inp, **cot}.items()}
    ref = oracle.attn_jvp_bwd_causal(*(fl[n][None] for n in NAMES), fl["dout"][None], fl["dtout"][None], w.scale,
                                     qrows=[], krows=keys)
    for n in ("dk", "dv", "dtk", "dtv"):
        err[n] = max_rel(got[n].reshape(-1, w.Lk, w.d)[h][keys].float().cpu().numpy(), ref[n][0])
    print(w.name, err)
    for n, e in err.items():
        assert e <= TOL, f"{n}: {e:.3e}"
    del inp, cot, got, o, to
    torch.cuda.empty_cache()
