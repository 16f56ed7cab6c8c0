"""Causal and packed (variable-length) forward against the fp64 masked
oracle, with the forward's bounds (O 1e-2, tO 2e-2, lse 1e-3 of max|ref|,
over rows that see at least one key); rows that see no key must be exact
zeros with lse = -inf.  Plus bit-exact agreement with the unmasked kernel
where the mask removes nothing."""
import numpy as np
import pytest
import torch

import attention_forward_mode_b200 as ajvp
import oracle
from attention_forward_mode_b200.workloads import WORKLOADS, custom, make_inputs, sample_rows
from gpu_common import TOL, gpu_inputs, max_rel

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "tq", "tk", "tv")
BOUND = TOL["bf16"]


def check(got, ref, rows_seen, what):
    o, to, lse = (x.float().cpu().numpy() if torch.is_tensor(x) else x for x in got)
    ro, rto, rlse = ref
    seen = rows_seen
    err = {"o": max_rel(o[seen], ro[seen]), "to": max_rel(to[seen], rto[seen]), "lse": max_rel(lse[seen], rlse[seen])}
    for key, e in err.items():
        assert e <= BOUND[key], f"{what}: {key} {e:.3e} > {BOUND[key]} ({err})"
    empty = ~seen
    if empty.any():
        assert np.all(o[empty] == 0) and np.all(to[empty] == 0) and np.all(np.isneginf(lse[empty])), what
    return err


@pytest.mark.parametrize("B,H,Lq,Lk", [(1, 1, 1, 1), (1, 2, 257, 257), (2, 3, 300, 300), (1, 2, 200, 333),
                                       (1, 2, 333, 200), (1, 2, 128, 64), (1, 1, 700, 1500)])
def test_causal_dense(B, H, Lq, Lk):
    w = custom(B, H, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=Lq * 3 + Lk)
    got = ajvp.attn_jvp_fwd_causal(*(inp[n] for n in NAMES), w.scale)
    torch.cuda.synchronize()
    ref = oracle.attn_jvp_causal(*(inp[n] for n in NAMES), w.scale)
    i = np.arange(Lq)[None, None, :]
    seen = np.broadcast_to(i + (Lk - Lq) >= 0, (B, H, Lq))
    print(w.name, check(got, ref, seen, w.name))


def test_causal_image_workload_sampled():
    w = WORKLOADS["image_selfattn_b2h12_l4096_d128"]
    inp = gpu_inputs(w)
    o, to, lse = ajvp.attn_jvp_fwd_causal(*(inp[n] for n in NAMES), w.scale)
    torch.cuda.synchronize()
    rows = sample_rows(w.Lq, 24)
    fl = {n: t.reshape(-1, t.shape[-2], t.shape[-1]) for n, t in inp.items()}
    for h in (0, 13, w.B * w.H - 1):
        for i in rows:
            r = oracle.attn_jvp(*(fl[n][h][i:i + 1][None] if n in ("q", "tq") else fl[n][h][:i + 1][None]
                                  for n in NAMES), w.scale)
            got = (o.reshape(-1, w.Lq, w.d)[h, i], to.reshape(-1, w.Lq, w.d)[h, i], lse.reshape(-1, w.Lq)[h, i])
            for g, rr, key in zip(got, r, ("o", "to", "lse")):
                e = max_rel(g.float().cpu().numpy(), rr[0, 0])
                assert e <= BOUND[key] * 2, (h, i, key, e)


def _packed_inputs(H, lq, lk, seed):
    g = torch.Generator().manual_seed(seed)
    Tq, Tk = sum(lq), sum(lk)
    x = {n: torch.randn((H, Tq if n in ("q", "tq") else Tk, 128), generator=g).to(torch.bfloat16).cuda()
         for n in NAMES}
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32, device="cuda")
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32, device="cuda")
    return x, cq, ck


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lq,lk", [([300, 1, 129, 0, 64], [200, 513, 7, 40, 0]),  # ragged, empty on either side
                                   ([1000, 250], [1000, 250]),
                                   ([64, 200, 77], [512, 512, 512])])                # text-like keys
def test_varlen(lq, lk, causal):
    H = 2
    x, cq, ck = _packed_inputs(H, lq, lk, seed=len(lq) + sum(lq))
    s = 128 ** -0.5
    got = ajvp.attn_jvp_fwd_varlen(*(x[n] for n in NAMES), cq, ck, max(lq), s, causal=causal)
    torch.cuda.synchronize()
    ref = oracle.attn_jvp_packed(*(x[n] for n in NAMES), s, cq.cpu().numpy(), ck.cpu().numpy(), causal)
    seen = np.zeros(sum(lq), dtype=bool)
    r0 = 0
    for a, b in zip(lq, lk):
        i = np.arange(a)
        seen[r0:r0 + a] = (i + (b - a) >= 0) if causal else (b > 0)
        seen[r0:r0 + a] &= b > 0
        r0 += a
    seen = np.broadcast_to(seen[None], (H, sum(lq)))
    print(lq, lk, causal, check(got, ref, seen, f"varlen causal={causal}"))


def test_unmasked_paths_agree_bitwise():
    # one packed sequence, no mask: the same arithmetic as attn_jvp_fwd (stores differ)
    w = custom(1, 3, 333, 517, 128)
    inp = gpu_inputs(w, seed=5)
    dense = ajvp.attn_jvp_fwd(*(inp[n] for n in NAMES), w.scale)
    x = {n: t[0] for n, t in inp.items()}
    cq = torch.tensor([0, w.Lq], dtype=torch.int32, device="cuda")
    ck = torch.tensor([0, w.Lk], dtype=torch.int32, device="cuda")
    packed = ajvp.attn_jvp_fwd_varlen(*(x[n] for n in NAMES), cq, ck, w.Lq, w.scale)
    # and the causal dense path against the causal packed path with one sequence
    cd = ajvp.attn_jvp_fwd_causal(*(inp[n] for n in NAMES), w.scale)
    cp = ajvp.attn_jvp_fwd_varlen(*(x[n] for n in NAMES), cq, ck, w.Lq, w.scale, causal=True)
    torch.cuda.synchronize()
    for a, b in zip(dense, packed):
        assert torch.equal(a[0], b)
    for a, b in zip(cd, cp):
        assert torch.equal(a[0], b)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("n", [32, 33, 64])
def test_many_short_sequences(n, causal):
    # n sequences of 1..300 tokens (two heads): the grid has many empty tiles.  Without
    # the mask, up to 32 sequences go out longest first (ranked inside the kernel), more
    # in the causal order
    rng = np.random.default_rng(n)
    lq = [int(v) for v in rng.integers(1, 300, size=n)]
    lk = [int(v) for v in rng.integers(1, 300, size=n)]
    x, cq, ck = _packed_inputs(2, lq, lk, seed=9)
    s = 0.1
    got = ajvp.attn_jvp_fwd_varlen(*(x[n_] for n_ in NAMES), cq, ck, max(lq), s, causal=causal)
    torch.cuda.synchronize()
    ref = oracle.attn_jvp_packed(*(x[n_] for n_ in NAMES), s, cq.cpu().numpy(), ck.cpu().numpy(), causal)
    if causal:
        seen = np.concatenate([np.arange(a) + (b - a) >= 0 for a, b in zip(lq, lk)])
    else:
        seen = np.ones(sum(lq), dtype=bool)
    check(got, ref, np.broadcast_to(seen[None], (2, sum(lq))), f"{n} short, causal={causal}")


def test_causal_video_workload_sampled():
    # the bench configuration of --entry causal: rows checked one by one on their visible prefix
    w = WORKLOADS["video_selfattn_b1h12_l32760_d128"]
    inp = gpu_inputs(w)
    o, to, lse = ajvp.attn_jvp_fwd_causal(*(inp[n] for n in NAMES), w.scale)
    torch.cuda.synchronize()
    rows = sample_rows(w.Lq, 16)
    fl = {n: t.reshape(-1, t.shape[-2], t.shape[-1]) for n, t in inp.items()}
    worst = {"o": 0.0, "to": 0.0, "lse": 0.0}
    for h in (0, w.B * w.H - 1):
        for i in rows:
            r = oracle.attn_jvp(*(fl[n][h][i:i + 1][None] if n in ("q", "tq") else fl[n][h][:i + 1][None]
                                  for n in NAMES), w.scale)
            got = (o.reshape(-1, w.Lq, w.d)[h, i], to.reshape(-1, w.Lq, w.d)[h, i], lse.reshape(-1, w.Lq)[h, i])
            for g, rr, key in zip(got, r, ("o", "to", "lse")):
                worst[key] = max(worst[key], max_rel(g.float().cpu().numpy(), rr[0, 0]))
    print(worst)
    for key, e in worst.items():
        assert e <= BOUND[key], (key, e)
    del inp, o, to, lse
    torch.cuda.empty_cache()


def test_varlen_bench_configuration_sampled():
    # the bench configuration of --entry varlen: the 12 heads' 32760 tokens as 8 sequences
    w = WORKLOADS["video_selfattn_b1h12_l32760_d128"]
    inp = gpu_inputs(w)
    cuts = np.sort(np.random.default_rng(0).choice(np.arange(1, w.Lq), size=7, replace=False))
    bounds = np.concatenate([[0], cuts, [w.Lq]]).astype(np.int64)
    cu = torch.tensor(bounds, dtype=torch.int32, device="cuda")
    x = {n: t[0] for n, t in inp.items()}
    o, to, lse = ajvp.attn_jvp_fwd_varlen(*(x[n] for n in NAMES), cu, cu, int(np.diff(bounds).max()), w.scale)
    torch.cuda.synchronize()
    worst = {"o": 0.0, "to": 0.0, "lse": 0.0}
    for h in (0, w.H - 1):
        for b in (0, 3, 7):
            a0, a1 = int(bounds[b]), int(bounds[b + 1])
            rows = sorted({a0, a1 - 1, (a0 + a1) // 2})
            ks = slice(a0, a1)
            for r in rows:
                ref = oracle.attn_jvp(*(x[n][h, r:r + 1][None] if n in ("q", "tq") else x[n][h, ks][None]
                                        for n in NAMES), w.scale)
                for g, rr, key in zip((o[h, r], to[h, r], lse[h, r]), ref, ("o", "to", "lse")):
                    worst[key] = max(worst[key], max_rel(g.float().cpu().numpy(), rr[0, 0]))
    print(worst)
    for key, e in worst.items():
        assert e <= BOUND[key], (key, e)
