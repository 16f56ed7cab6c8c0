"""The backward's dQ/dtQ and dK/dtK kernels as CTA pairs (two CTAs of a
cluster share each tensor-core product, cta_group::2) against the fp64
backward oracle, and against the one-CTA form of the same kernels.

The pair form runs for the unmasked kernels without a split key side, so
the key-side cases here pass a workspace of the statistics size only
(bwd_workspace_bytes(B, H, Lq)), which keeps the key side unsplit.  Shapes
with an odd number of 128-row tiles leave the last pair's second CTA past
the end of the rows: it takes its part in the products and stores nothing.
Bound on max|err| / max|ref|: 2e-2, as for the other backward tests.  The
two forms add each tile's G2 products in a different order, so they agree
to rounding (bound 1e-2 relative to the largest gradient entry), not bit
for bit."""
import pytest
import torch

import attention_forward_mode_b200 as ajvp
import oracle
from attention_forward_mode_b200.workloads import custom, make_cotangents
from gpu_common import gpu_inputs, max_rel

pytestmark = pytest.mark.gpu

TOL = 2e-2
NAMES = ("q", "k", "v", "tq", "tk", "tv")
GRADS = ("dq", "dk", "dv", "dtq", "dtk", "dtv")


def run(inp, cot, scale, pairs, step=None):
    B, H, Lq, _ = inp["q"].shape
    o, to, lse, mu = ajvp.attn_jvp_fwd_stats(*(inp[n] for n in NAMES), scale)
    ws = torch.empty(ajvp.bwd_workspace_bytes(B, H, Lq), dtype=torch.uint8, device="cuda")
    ajvp.set_bwd_pairs(pairs)
    try:
        if step is None:
            g = ajvp.attn_jvp_bwd(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], scale,
                                  workspace=ws)
        else:
            g = {n: torch.zeros_like(inp["q"] if n in ("dq", "dtq") else inp["k"]) for n in GRADS}
            for s in range(4):
                ajvp.attn_jvp_bwd(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], scale,
                                  grads=g, workspace=ws, step=s)
        torch.cuda.synchronize()
    finally:
        ajvp.set_bwd_pairs(ajvp.DEFAULT_BWD_PAIRS)
    assert ajvp.check_device_status() == ajvp.AJVP_OK
    return g


# (1, 1, 1, 1): one row tile on each side (the pair's second CTA idle);
# 129 x 127: two row tiles, ragged; 300 x 700: three query tiles and six key
# tiles; 257 x 1000: three query tiles, eight key tiles; 640 x 384, H = 3:
# five query tiles, three key tiles over several heads
@pytest.mark.parametrize("B,H,Lq,Lk", [(1, 1, 1, 1), (1, 2, 129, 127), (2, 3, 300, 700), (1, 1, 257, 1000),
                                       (1, 3, 640, 384)])
def test_pairs_against_oracle_and_single(B, H, Lq, Lk):
    w = custom(B, H, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=Lq + 3 * Lk)
    cot = make_cotangents(w, seed=Lq + 5 * Lk, device="cuda")
    pair = run(inp, cot, w.scale, True)
    single = run(inp, cot, w.scale, False)
    ref = oracle.attn_jvp_bwd(*(inp[n] for n in NAMES), cot["dout"], cot["dtout"], w.scale)
    err = {n: max_rel(pair[n].float().cpu().numpy(), ref[n]) for n in GRADS}
    err1 = {n: max_rel(single[n].float().cpu().numpy(), ref[n]) for n in GRADS}
    print(w.name, "pairs", err, "single", err1)
    for n in GRADS:
        assert err[n] <= TOL, f"{w.name}: {n} (pairs) max-rel error {err[n]:.3e} > {TOL}"
        assert err1[n] <= TOL, f"{w.name}: {n} (single) max-rel error {err1[n]:.3e} > {TOL}"
        # the value side (dv, dtv) does not use pairs: identical
        if n in ("dv", "dtv"):
            assert torch.equal(pair[n], single[n]), n
        else:
            d = (pair[n].float() - single[n].float()).abs().max().item()
            scale = single[n].float().abs().max().item()
            assert d <= 1e-2 * max(scale, 1e-30), (n, d, scale)


def test_pairs_deterministic_and_stepwise():
    w = custom(1, 2, 520, 600, 128)
    inp = gpu_inputs(w, seed=21)
    cot = make_cotangents(w, seed=22, device="cuda")
    a = run(inp, cot, w.scale, True)
    b = run(inp, cot, w.scale, True)
    c = run(inp, cot, w.scale, True, step="each")
    for n in GRADS:
        assert torch.equal(a[n], b[n]), n
        assert torch.equal(a[n], c[n]), n


def test_pairs_zero_cotangents():
    w = custom(1, 2, 300, 260, 128)
    inp = gpu_inputs(w, seed=23)
    cot = {n: torch.zeros((w.B, w.H, w.Lq, w.d), dtype=torch.bfloat16, device="cuda") for n in ("dout", "dtout")}
    got = run(inp, cot, w.scale, True)
    for n in GRADS:
        assert torch.count_nonzero(got[n]).item() == 0, n


def test_pairs_video_workload_sampled():
    # the video self-attention configuration (12 heads x 32760, 256 row tiles per
    # head: 128 pairs) with pairs: sampled query rows of three heads and keys of one
    # head against the oracle, and every gradient close to the one-CTA form
    from attention_forward_mode_b200.workloads import WORKLOADS, sample_rows
    w = WORKLOADS["video_selfattn_b1h12_l32760_d128"]
    inp = gpu_inputs(w)
    cot = make_cotangents(w, device="cuda")
    got = run(inp, cot, w.scale, True)
    single = run(inp, cot, w.scale, False)
    err = {}
    rows = sample_rows(w.Lq, 12)
    for h in (0, 7, w.B * w.H - 1):
        fl = {n: t.reshape(-1, t.shape[-2], t.shape[-1])[h] for n, t in {**inp, **cot}.items()}
        ref = oracle.attn_jvp_bwd(*(fl[n][None] for n in NAMES), fl["dout"][None], fl["dtout"][None], w.scale,
                                  qrows=rows, krows=[])
        for n in ("dq", "dtq"):
            e = max_rel(got[n].reshape(-1, w.Lq, w.d)[h][rows].float().cpu().numpy(), ref[n][0])
            err[n] = max(err.get(n, 0.0), e)
    h = 5
    keys = sample_rows(w.Lk, 8, seed=1)
    fl = {n: t.reshape(-1, t.shape[-2], t.shape[-1])[h].cpu() for n, t in {**inp, **cot}.items()}
    ref = oracle.attn_jvp_bwd(*(fl[n][None] for n in NAMES), fl["dout"][None], fl["dtout"][None], w.scale,
                              qrows=[], krows=keys)
    for n in ("dk", "dtk"):
        err[n] = max_rel(got[n].reshape(-1, w.Lk, w.d)[h][keys].float().cpu().numpy(), ref[n][0])
    print(w.name, err)
    for n, e in err.items():
        assert e <= TOL, f"{n}: {e:.3e}"
    for n in ("dq", "dtq", "dk", "dtk"):
        d = (got[n].float() - single[n].float()).abs().max().item()
        assert d <= 1e-2 * single[n].float().abs().max().item(), (n, d)
    del inp, cot, got, single
    torch.cuda.empty_cache()
