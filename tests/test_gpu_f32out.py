"""attn_jvp_fwd_f32out (bf16 inputs, fp32 outputs, split-bf16 probability
operands) against the fp64 oracle.

Bound on max|err| / max|ref| for O and tO: 1e-4, the fp32 bound, at every
key length (the tensor cores' accumulation truncates each product to the
accumulator's precision, which over tens of thousands of keys biased the
sums toward zero; the kernel folds its accumulators into the fp32 outputs
every 32 key tiles, so the error no longer grows with Lk).  lse: 1e-5.  Also:
the variant's errors must sit at least 10x below those of the bf16-output
entry point on the same inputs (the point of the variant: BF16 JVP error is
much larger than BF16 output error), the error must not grow with the key
length, and rows whose max keeps rising (rescales between folds) must stay
within the bound."""
import numpy as np
import pytest
import torch

import attention_forward_mode_b200 as ajvp
import oracle
from attention_forward_mode_b200.workloads import WORKLOADS, custom, sample_rows
from gpu_common import compare_full, gpu_inputs, max_rel

pytestmark = pytest.mark.gpu


def tol(Lk):
    return {"o": 1e-4, "to": 1e-4, "lse": 1e-5}


def run_f32out(inp, scale):
    out = ajvp.attn_jvp_fwd_f32out(inp["q"], inp["k"], inp["v"], inp["tq"], inp["tk"], inp["tv"], scale)
    torch.cuda.synchronize()
    assert out[0].dtype == torch.float32 and out[1].dtype == torch.float32
    return out


def check(err, what, Lk):
    bound = tol(Lk)
    for key in ("o", "to", "lse"):
        assert err[key] <= bound[key], f"{what}: {key} max-rel error {err[key]:.3e} > {bound[key]:.1e} ({err})"


@pytest.mark.parametrize("B,H,Lq,Lk", [(1, 1, 1, 1), (1, 2, 129, 127), (2, 3, 300, 700), (1, 1, 257, 4097)])
def test_shapes_full(B, H, Lq, Lk):
    w = custom(B, H, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=Lq + Lk)
    err = compare_full(w, inp, run_f32out(inp, w.scale))
    print(w.name, err)
    check(err, w.name, Lk)


@pytest.mark.parametrize("name", ["image_selfattn_b2h12_l4096_d128", "video_selfattn_b1h12_l32760_d128",
                                  "video_crossattn_b1h40_lq32760_lk512_d128",
                                  "video_selfattn_large_b1h40_l75600_d128"])
def test_workloads_sampled(name):
    w = WORKLOADS[name]
    inp = gpu_inputs(w)
    out = run_f32out(inp, w.scale)
    bh = w.B * w.H
    heads = sorted({0, bh // 2, bh - 1})
    rows = sample_rows(w.Lq, 24)
    idx = torch.tensor(rows, device="cuda")
    fl = {n: t.reshape(-1, t.shape[-2], t.shape[-1]) for n, t in inp.items()}
    got = [[], [], []]
    ref = [[], [], []]
    for h in heads:
        q = fl["q"][h].index_select(0, idx).cpu()
        tq = fl["tq"][h].index_select(0, idx).cpu()
        k, v, tk, tv = (fl[n][h].cpu() for n in ("k", "v", "tk", "tv"))
        r = oracle.attn_jvp(q[None], k[None], v[None], tq[None], tk[None], tv[None], w.scale)
        for i in range(3):
            ref[i].append(r[i][0])
        got[0].append(out[0].reshape(-1, w.Lq, w.d)[h].index_select(0, idx).cpu().numpy())
        got[1].append(out[1].reshape(-1, w.Lq, w.d)[h].index_select(0, idx).cpu().numpy())
        got[2].append(out[2].reshape(-1, w.Lq)[h].index_select(0, idx).cpu().numpy())
    err = {k: max_rel(np.stack(got[i]), np.stack(ref[i])) for i, k in enumerate(("o", "to", "lse"))}
    print(name, err)
    check(err, name, w.Lk)
    del inp, out
    torch.cuda.empty_cache()


def test_tangent_error_far_below_bf16_path():
    w = custom(1, 4, 640, 2048, 128)
    inp = gpu_inputs(w, seed=21)
    e32 = compare_full(w, inp, run_f32out(inp, w.scale))
    o, to, lse = ajvp.attn_jvp_fwd(inp["q"], inp["k"], inp["v"], inp["tq"], inp["tk"], inp["tv"], w.scale)
    torch.cuda.synchronize()
    e16 = compare_full(w, inp, (o, to, lse))
    print("f32out", e32, "bf16", e16)
    assert e32["to"] * 10 <= e16["to"]
    assert e32["o"] * 10 <= e16["o"]


def _one_head_full(Lk, seed, key_ramp=None):
    w = custom(1, 1, 256, Lk, 128)
    inp = gpu_inputs(w, seed=seed)
    if key_ramp is not None:
        f = torch.linspace(key_ramp[0], key_ramp[1], Lk, device="cuda")[None, None, :, None]
        inp["k"] = (inp["k"].float() * f).to(torch.bfloat16)
    return w, compare_full(w, inp, run_f32out(inp, w.scale))


def test_error_flat_in_key_length():
    # 2 key tiles (no fold) against 1024 key tiles (31 folds): without the folds the
    # truncated accumulation grew the error about linearly (4e-6 -> 2e-4)
    _, short = _one_head_full(128, 41)
    w, long = _one_head_full(65536, 42)
    print("Lk 128", short, "Lk 65536", long)
    check(long, w.name, w.Lk)
    for key in ("o", "to"):
        assert long[key] <= 3 * short[key] + 3e-6, (key, short, long)


def test_rising_row_max_rescales_between_folds():
    # key rows scaled by a ramp 0.25 -> 3: each row's max keeps rising along the keys, so
    # the reference max is raised after folds have happened (the folded sums are rescaled)
    w, err = _one_head_full(32760 + 37, 43, key_ramp=(0.25, 3.0))
    print(w.name, "ramped keys", err)
    check(err, w.name, w.Lk)


def test_zero_tangent_exact_zero():
    w = custom(1, 2, 200, 300, 128)
    inp = gpu_inputs(w, seed=2)
    for n in ("tq", "tk", "tv"):
        inp[n].zero_()
    _, to, _ = run_f32out(inp, w.scale)
    assert torch.count_nonzero(to).item() == 0


def _masked_err(got, ref, seen):
    o, to, lse = (x.float().cpu().numpy() for x in got)
    ro, rto, rlse = ref
    err = {"o": max_rel(o[seen], ro[seen]), "to": max_rel(to[seen], rto[seen]),
           "lse": max_rel(lse[seen], rlse[seen])}
    empty = ~seen
    if empty.any():
        assert np.all(o[empty] == 0) and np.all(to[empty] == 0) and np.all(np.isneginf(lse[empty]))
    return err


@pytest.mark.parametrize("B,H,Lq,Lk", [(1, 2, 200, 200), (1, 2, 129, 300), (1, 1, 333, 130)])
def test_causal_against_masked_oracle(B, H, Lq, Lk):
    # the causal mask of attn_jvp_fwd_causal; rows that see no key: zeros, lse = -inf
    w = custom(B, H, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=2 * Lq + Lk)
    names = ("q", "k", "v", "tq", "tk", "tv")
    got = ajvp.attn_jvp_fwd_f32out_causal(*(inp[n] for n in names), w.scale)
    bf = ajvp.attn_jvp_fwd_causal(*(inp[n] for n in names), w.scale)
    torch.cuda.synchronize()
    assert got[0].dtype == torch.float32
    ref = oracle.attn_jvp_causal(*(inp[n] for n in names), w.scale)
    i = np.arange(Lq)
    seen = np.broadcast_to((i + (Lk - Lq) >= 0)[None, None], (B, H, Lq))
    err = _masked_err(got, ref, seen)
    err_bf = _masked_err(bf, ref, seen)
    print(w.name, err, err_bf)
    check(err, w.name, Lk)
    assert err["to"] * 10 <= err_bf["to"], (err, err_bf)


def test_causal_long_keys_fold():
    # long enough that the later query tiles' key ranges pass several folds (every 32
    # tiles of 64 keys), with a ragged tail on both sides; rows checked: a sample that
    # includes the first and last tiles
    B, H, Lq, Lk = 1, 2, 4500, 4600
    w = custom(B, H, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=61)
    names = ("q", "k", "v", "tq", "tk", "tv")
    got = ajvp.attn_jvp_fwd_f32out_causal(*(inp[n] for n in names), w.scale)
    torch.cuda.synchronize()
    rows = sample_rows(Lq, 160, seed=3)
    fl = {n: t.reshape(-1, t.shape[-2], t.shape[-1]) for n, t in inp.items()}
    err = {"o": 0.0, "to": 0.0, "lse": 0.0}
    for h in range(B * H):
        # each sampled row alone against its visible keys (causal, bottom-right aligned)
        ref = oracle.attn_jvp_causal(*(fl[n][h][None].cpu() for n in names), w.scale)
        for i, key in enumerate(("o", "to", "lse")):
            g = got[i].reshape(-1, Lq, *(() if key == "lse" else (128,)))[h][rows].cpu().numpy()
            err[key] = max(err[key], max_rel(g, ref[i][0][rows]))
    print(w.name, "causal, long keys", err)
    check(err, w.name, Lk)


def test_varlen_long_sequences_fold():
    # packed sequences long enough to fold (2100 and 4200 keys) next to short ones, so
    # that the folds' row guard keeps a tile's overhang out of the next sequence
    H, lq, lk = 2, [700, 90, 300], [4200, 130, 2100]
    g = torch.Generator().manual_seed(78)
    names = ("q", "k", "v", "tq", "tk", "tv")
    x = {n: torch.randn((H, sum(lq) if n in ("q", "tq") else sum(lk), 128), generator=g).to(torch.bfloat16).cuda()
         for n in names}
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32, device="cuda")
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32, device="cuda")
    s = 128 ** -0.5
    for causal in (False, True):
        got = ajvp.attn_jvp_fwd_f32out_varlen(*(x[n] for n in names), cq, ck, max(lq), s, causal=causal)
        torch.cuda.synchronize()
        ref = oracle.attn_jvp_packed(*(x[n] for n in names), s, cq.cpu().numpy(), ck.cpu().numpy(), causal)
        seen = np.ones(sum(lq), dtype=bool)  # Lq <= Lk in every sequence: every row sees a key
        err = _masked_err(got, ref, np.broadcast_to(seen[None], (H, sum(lq))))
        print("varlen long, causal", causal, err)
        check(err, f"varlen long causal={causal}", max(lk))


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_against_masked_oracle(causal):
    H, lq, lk = 2, [300, 1, 129, 0, 64], [200, 513, 7, 40, 0]
    g = torch.Generator().manual_seed(77)
    names = ("q", "k", "v", "tq", "tk", "tv")
    x = {n: torch.randn((H, sum(lq) if n in ("q", "tq") else sum(lk), 128), generator=g).to(torch.bfloat16).cuda()
         for n in names}
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32, device="cuda")
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32, device="cuda")
    s = 128 ** -0.5
    got = ajvp.attn_jvp_fwd_f32out_varlen(*(x[n] for n in names), cq, ck, max(lq), s, causal=causal)
    torch.cuda.synchronize()
    assert got[0].dtype == torch.float32
    ref = oracle.attn_jvp_packed(*(x[n] for n in names), s, cq.cpu().numpy(), ck.cpu().numpy(), causal)
    seen = np.zeros(sum(lq), dtype=bool)
    r0 = 0
    for a, b in zip(lq, lk):
        i = np.arange(a)
        seen[r0:r0 + a] = ((i + (b - a) >= 0) if causal else np.full(a, True)) & (b > 0)
        r0 += a
    err = _masked_err(got, ref, np.broadcast_to(seen[None], (H, sum(lq))))
    print(causal, err)
    check(err, f"varlen causal={causal}", max(lk))
