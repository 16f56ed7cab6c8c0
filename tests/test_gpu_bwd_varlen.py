"""attn_jvp_bwd_varlen (the backward of the packed variable-length forward,
optionally causal inside each sequence) against the fp64 masked backward
oracle on the same bf16 inputs, with the unmasked backward's bound (2e-2 of
max|ref| per gradient); gradients of rows that see no key, and of keys that
no row sees, must be exact zeros.  Plus bit-exact agreement with the dense
entry points for one packed sequence."""
import numpy as np
import pytest
import torch

import attention_forward_mode_b200 as ajvp
import oracle
from attention_forward_mode_b200.workloads import WORKLOADS, custom, make_cotangents
from gpu_common import gpu_inputs, max_rel

pytestmark = pytest.mark.gpu

TOL = 2e-2
NAMES = ("q", "k", "v", "tq", "tk", "tv")
GRADS = ("dq", "dk", "dv", "dtq", "dtk", "dtv")


def _packed(H, lq, lk, seed):
    g = torch.Generator().manual_seed(seed)
    Tq, Tk = sum(lq), sum(lk)
    x = {n: torch.randn((H, Tq if n in ("q", "tq", "dout", "dtout") else Tk, 128),
                        generator=g).to(torch.bfloat16).cuda()
         for n in NAMES + ("dout", "dtout")}
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32, device="cuda")
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32, device="cuda")
    return x, cq, ck


def _run(x, cq, ck, lq, lk, s, causal, with_forward=False):
    o, to, lse, mu = ajvp.attn_jvp_fwd_varlen_stats(*(x[n] for n in NAMES), cq, ck, max(lq), s, causal=causal)
    g = ajvp.attn_jvp_bwd_varlen(*(x[n] for n in NAMES), o, to, lse, mu, x["dout"], x["dtout"], cq, ck, max(lq),
                                 max(lk), s, causal=causal)
    torch.cuda.synchronize()
    assert ajvp.check_device_status() == ajvp.AJVP_OK
    return (g, o, to) if with_forward else g


def _statistics_leak(x, o, to, lq, lk, s, causal):
    """First-order effect on the gradients of the forward's bf16 outputs.

    The backward's row statistics a_i = <dtO_i, O_i> and
    D_i = <dO_i, O_i> + <dtO_i, tO_i> - a_i mu_i are formed from the O, tO the
    forward returned (bf16, as FlashAttention forms D from its bf16 O), so they
    carry deviations da_i, dD_i from their exact values.  Through
    S_bar = P (B + A (u - mu) - a u - D) and dS_bar = P (A - a) these give
    dS_bar' = -P (da u + dD), ddS_bar = -P da, hence
    dq' = s (dS_bar' K + ddS_bar tK), dtq' = s ddS_bar K,
    dk' = s (dS_bar'^T Q + ddS_bar^T tQ), dtk' = s ddS_bar^T Q (dv, dtv do not
    use them).  In a row that sees many keys P spreads and the effect averages
    out; in a row that sees one or a few keys it enters undiluted.  Computed
    in fp64 from the inputs, the exact softmax and the returned O, tO."""
    f = {n: t.double().cpu().numpy() for n, t in {**x, "o": o, "to": to}.items()}
    H = f["q"].shape[0]
    leak = {n: np.zeros_like(f["q"] if n in ("dq", "dtq") else f["k"]) for n in ("dq", "dtq", "dk", "dtk")}
    r0 = c0 = 0
    for a, b in zip(lq, lk):
        if a and b:
            rq, rk = slice(r0, r0 + a), slice(c0, c0 + b)
            i, j = np.arange(a)[:, None], np.arange(b)[None, :]
            vis = (j <= i + (b - a)) if causal else np.ones((a, b), dtype=bool)
            for h in range(H):
                q, tq = f["q"][h, rq], f["tq"][h, rq]
                k, tk, v, tv = f["k"][h, rk], f["tk"][h, rk], f["v"][h, rk], f["tv"][h, rk]
                S = np.where(vis, s * q @ k.T, -np.inf)
                m = S.max(1, keepdims=True)
                P = np.where(vis, np.exp(S - np.where(np.isfinite(m), m, 0.0)), 0.0)
                den = P.sum(1, keepdims=True)
                P = np.divide(P, den, out=np.zeros_like(P), where=den > 0)
                u = s * (tq @ k.T + q @ tk.T)
                mu = (P * u).sum(1)
                O = P @ v
                tO = (P * (u - mu[:, None])) @ v + P @ tv
                do, dto = f["dout"][h, rq], f["dtout"][h, rq]
                da = np.einsum("id,id->i", dto, f["o"][h, rq] - O)
                dD = np.einsum("id,id->i", do, f["o"][h, rq] - O) + np.einsum("id,id->i", dto, f["to"][h, rq] - tO)
                dD -= da * mu
                dsb = -P * (da[:, None] * u + dD[:, None])
                ddsb = -P * da[:, None]
                leak["dq"][h, rq] = s * (dsb @ k + ddsb @ tk)
                leak["dtq"][h, rq] = s * ddsb @ k
                leak["dk"][h, rk] = s * (dsb.T @ q + ddsb.T @ tq)
                leak["dtk"][h, rk] = s * ddsb.T @ q
        r0 += a
        c0 += b
    return leak


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lq,lk", [([300, 1, 129, 0, 64], [200, 513, 7, 40, 0]),  # ragged, empty on either side
                                   ([1000, 250], [1000, 250]),
                                   ([64, 200, 77], [512, 512, 512]),               # text-like keys
                                   ([130, 127, 256], [129, 300, 2])])
def test_varlen(lq, lk, causal):
    H = 2
    x, cq, ck = _packed(H, lq, lk, seed=len(lq) + sum(lq) + sum(lk))
    s = 128 ** -0.5
    got, o, to = _run(x, cq, ck, lq, lk, s, causal, with_forward=True)
    ref = oracle.attn_jvp_bwd_packed(*(x[n] for n in NAMES), x["dout"], x["dtout"], s, cq.cpu().numpy(),
                                     ck.cpu().numpy(), causal)
    err = {n: max_rel(got[n].float().cpu().numpy(), ref[n]) for n in GRADS}
    print(lq, lk, causal, err)
    # the relative bound, plus (for the gradients that use the row statistics) the
    # first-order effect of the forward's bf16 outputs on them, which rows seeing
    # only a few keys (causal rows near a sequence's start when Lq > Lk) feel undiluted
    leak = _statistics_leak(x, o, to, lq, lk, s, causal)
    for n in GRADS:
        g = got[n].double().cpu().numpy()
        excess = np.abs(g - ref[n]) - (1.05 * np.abs(leak[n]) if n in leak else 0.0)
        e = float(excess.max()) / float(np.abs(ref[n]).max())
        assert e <= TOL, f"{n}: max-rel error {err[n]:.3e}, {e:.3e} beyond the bf16-statistics effect ({err})"
    # rows that see no key and keys no row sees: exact zeros
    host = {n: got[n].float().cpu().numpy() for n in GRADS}
    r0 = c0 = 0
    for a, b in zip(lq, lk):
        i = np.arange(a)
        blind = (i + (b - a) < 0) if causal else np.full(a, b == 0)
        blind |= b == 0
        for n in ("dq", "dtq"):
            assert np.all(host[n][:, r0:r0 + a][:, blind] == 0), (a, b, n)
        if a == 0:
            for n in ("dk", "dv", "dtk", "dtv"):
                assert np.all(host[n][:, c0:c0 + b] == 0), (a, b, n)
        r0 += a
        c0 += b


@pytest.mark.parametrize("causal", [False, True])
def test_one_sequence_equals_dense(causal):
    # one packed sequence: the dense kernels' arithmetic, bit for bit (the packed
    # epilogue stores rows directly instead of through the tensor-store unit; the
    # dense call gets the statistics-only workspace, so its key side does not split,
    # and runs its dQ / dK kernels one CTA per row tile, as the packed ones do: the
    # CTA-pair form adds each tile's products in another order)
    w = custom(1, 3, 333, 517, 128)
    inp = gpu_inputs(w, seed=41)
    cot = make_cotangents(w, seed=42, device="cuda")
    fwd = ajvp.attn_jvp_fwd_causal_stats if causal else ajvp.attn_jvp_fwd_stats
    bwd = ajvp.attn_jvp_bwd_causal if causal else ajvp.attn_jvp_bwd
    o, to, lse, mu = fwd(*(inp[n] for n in NAMES), w.scale)
    ws = torch.empty(ajvp.bwd_workspace_bytes(w.B, w.H, w.Lq), dtype=torch.uint8, device="cuda")
    ajvp.set_bwd_pairs(False)
    try:
        dense = bwd(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], w.scale, workspace=ws)
        torch.cuda.synchronize()
    finally:
        ajvp.set_bwd_pairs(ajvp.DEFAULT_BWD_PAIRS)
    x = {n: t[0] for n, t in {**inp, **cot}.items()}
    cq = torch.tensor([0, w.Lq], dtype=torch.int32, device="cuda")
    ck = torch.tensor([0, w.Lk], dtype=torch.int32, device="cuda")
    got = _run(x, cq, ck, [w.Lq], [w.Lk], w.scale, causal)
    for n in GRADS:
        assert torch.equal(got[n], dense[n][0]), n


def test_single_key_sequence():
    # a sequence with one key: P = 1, O = V_0 and tO = tV_0 exactly, so the exact
    # gradients with respect to its queries, K_0 and tK_0 vanish.  The kernels' row
    # statistic D_i = <dO, O> + <dtO, tO> - a mu is formed from the forward's bf16
    # outputs, whose deviation dD_i (the forward's bf16 P.*dS operand leaves tO_i off
    # tV_0) enters S_bar = -dD_i undiluted: |dq_i| <= s |dD_i| max|K_0| and
    # |dk_0| <= s sum_i |dD_i| |Q_i| per column (a_i is exact: O_i = bf16(V_0) = V_0).
    # dv_0 = sum_i dO_i and dtv_0 = sum_i dtO_i are not affected: oracle bound.
    H, lq, lk = 2, [200, 150], [300, 1]
    x, cq, ck = _packed(H, lq, lk, seed=44)
    s = 128 ** -0.5
    o, to, lse, mu = ajvp.attn_jvp_fwd_varlen_stats(*(x[n] for n in NAMES), cq, ck, max(lq), s)
    g = ajvp.attn_jvp_bwd_varlen(*(x[n] for n in NAMES), o, to, lse, mu, x["dout"], x["dtout"], cq, ck, max(lq),
                                 max(lk), s)
    torch.cuda.synchronize()
    ref = oracle.attn_jvp_bwd_packed(*(x[n] for n in NAMES), x["dout"], x["dtout"], s, cq.cpu().numpy(),
                                     ck.cpu().numpy(), False)
    f64 = {n: t.double().cpu().numpy() for n, t in {**x, "o": o, "to": to}.items()}
    got = {n: t.double().cpu().numpy() for n, t in g.items()}
    rows = slice(lq[0], lq[0] + lq[1])
    key = lk[0]
    for h in range(H):
        dD = (np.einsum("id,id->i", f64["dout"][h, rows], f64["o"][h, rows] - f64["v"][h, key])
              + np.einsum("id,id->i", f64["dtout"][h, rows], f64["to"][h, rows] - f64["tv"][h, key]))
        kmax = np.abs(f64["k"][h, key]).max()
        bq = s * np.abs(dD) * kmax * 1.01 + 1e-4
        assert np.all(np.abs(got["dq"][h, rows]).max(1) <= bq), h
        bk = s * (np.abs(dD)[:, None] * np.abs(f64["q"][h, rows])).sum(0) * 1.01 + 1e-3
        assert np.all(np.abs(got["dk"][h, key]) <= bk), h
        assert np.abs(got["dtq"][h, rows]).max() <= 1e-3 and np.abs(got["dtk"][h, key]).max() <= 1e-2, h
        print(h, np.abs(got["dk"][h, key]).max(), bk.max())
    # everything else, and dv_0, dtv_0, to the relative bound
    for n in GRADS:
        r = ref[n].copy()
        gg = got[n].copy()
        if n in ("dq", "dtq"):
            r[:, rows] = gg[:, rows] = 0.0
        elif n in ("dk", "dtk"):
            r[:, key] = gg[:, key] = 0.0
        assert max_rel(gg, r) <= TOL, n


def test_no_query_rows_zeroes_key_gradients():
    H, lk = 2, [100, 37]
    x, cq, ck = _packed(H, [0, 0], lk, seed=43)
    s = 128 ** -0.5
    grads = {n: torch.full_like(x["q"] if n in ("dq", "dtq") else x["k"], 7.0) for n in GRADS}
    o = torch.empty_like(x["q"])
    lse = torch.empty((H, 0), dtype=torch.float32, device="cuda")
    g = ajvp.attn_jvp_bwd_varlen(*(x[n] for n in NAMES), o, o.clone(), lse, lse.clone(), x["dout"], x["dtout"], cq,
                                 ck, 0, max(lk), s, grads=grads)
    torch.cuda.synchronize()
    for n in ("dk", "dv", "dtk", "dtv"):
        assert torch.count_nonzero(g[n]).item() == 0, n


def test_varlen_bench_configuration_sampled():
    # the 12 heads' 32760 video tokens as 8 packed sequences (the forward's --entry varlen
    # configuration): dQ, dtQ rows of three sequences one by one, and the key-side
    # gradients of a few keys of two sequences (each needs its own sequence's rows only)
    w = WORKLOADS["video_selfattn_b1h12_l32760_d128"]
    inp = gpu_inputs(w)
    cot = make_cotangents(w, device="cuda")
    cuts = np.sort(np.random.default_rng(0).choice(np.arange(1, w.Lq), size=7, replace=False))
    bounds = np.concatenate([[0], cuts, [w.Lq]]).astype(np.int64)
    cu = torch.tensor(bounds, dtype=torch.int32, device="cuda")
    x = {n: t[0] for n, t in {**inp, **cot}.items()}
    lens = np.diff(bounds).tolist()
    got = _run(x, cu, cu, lens, lens, w.scale, False)
    err = {n: 0.0 for n in GRADS}
    for h in (0, w.H - 1):
        for b in (0, 3, 7):
            a0, a1 = int(bounds[b]), int(bounds[b + 1])
            sl = slice(a0, a1)
            rows = sorted({0, a1 - a0 - 1, (a1 - a0) // 2, min(127, a1 - a0 - 1), min(128, a1 - a0 - 1)})
            keys = rows if b != 3 else []
            one = {n: x[n][h, sl][None].cpu() for n in x}
            ref = oracle.attn_jvp_bwd_packed(*(one[n] for n in NAMES), one["dout"], one["dtout"], w.scale,
                                             [0, a1 - a0], [0, a1 - a0], False, qrows=rows, krows=keys)
            for n in ("dq", "dtq"):
                g = got[n][h, sl][rows].float().cpu().numpy()
                err[n] = max(err[n], max_rel(g, ref[n][0]))
            for n in ("dk", "dv", "dtk", "dtv"):
                if keys:
                    g = got[n][h, sl][keys].float().cpu().numpy()
                    err[n] = max(err[n], max_rel(g, ref[n][0]))
    print(err)
    for n, e in err.items():
        assert e <= TOL, (n, e)
    del inp, cot, got, x
    torch.cuda.empty_cache()
