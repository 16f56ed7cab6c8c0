"""The unmasked backward with the key side split over the query range (short
key sequences: cross-attention to a few hundred tokens).  With a workspace of
attn_jvp_bwd_workspace_bytes_split bytes the dK, dtK and dV, dtV kernels cut
the streamed query tiles into parts, write fp32 partial sums and a reduction
adds them up in part order.  Held to the unsplit backward's bound against the
fp64 oracle (2e-2 of max|ref| per gradient), bit-exact from run to run, and
close to the unsplit kernels (which round the same fp32 sums once, in another
order)."""
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


def _bwd(w, inp, cot, split, step=None, grads=None):
    o, to, lse, mu = ajvp.attn_jvp_fwd_stats(*(inp[n] for n in NAMES), w.scale)
    nbytes = ajvp.bwd_workspace_bytes(w.B, w.H, w.Lq, w.Lk if split else None)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    g = ajvp.attn_jvp_bwd(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], w.scale,
                          workspace=ws, grads=grads, step=step)
    torch.cuda.synchronize()
    assert ajvp.check_device_status() == ajvp.AJVP_OK
    return g


@pytest.mark.parametrize("B,H,Lq,Lk", [(1, 2, 3000, 300),   # 16 parts of 3 query tiles, the last one of 2
                                       (2, 1, 1000, 77),    # one ragged key tile per head, 16 one-tile parts
                                       (1, 3, 700, 513)])   # a one-key last tile, the last part one ragged tile
def test_split_against_oracle(B, H, Lq, Lk):
    assert ajvp.bwd_workspace_bytes(B, H, Lq, Lk) > ajvp.bwd_workspace_bytes(B, H, Lq), "no split at this shape"
    w = custom(B, H, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=Lq + Lk)
    cot = make_cotangents(w, seed=2 * Lq + Lk, device="cuda")
    got = _bwd(w, inp, cot, split=True)
    ref = oracle.attn_jvp_bwd(*(inp[n] for n in NAMES), cot["dout"], cot["dtout"], w.scale)
    err = {n: max_rel(got[n].float().cpu().numpy(), ref[n]) for n in GRADS}
    print(w.name, err)
    for n, e in err.items():
        assert e <= TOL, f"{w.name}: {n} max-rel error {e:.3e} > {TOL} ({err})"


def test_split_many_key_tiles_sampled():
    # 24 heads x 4 key tiles = 96 key-side CTAs: 3 parts of 22 query tiles (the last
    # part 21, one of them ragged); sampled rows and keys on three heads
    w = custom(1, 24, 4100, 512, 128)
    assert ajvp.bwd_workspace_bytes(w.B, w.H, w.Lq, w.Lk) > ajvp.bwd_workspace_bytes(w.B, w.H, w.Lq)
    inp = gpu_inputs(w, seed=16)
    cot = make_cotangents(w, seed=17, device="cuda")
    got = _bwd(w, inp, cot, split=True)
    rows, keys = sample_rows(w.Lq, 10), sample_rows(w.Lk, 12, seed=2)
    err = {n: 0.0 for n in GRADS}
    for h in (0, 11, 23):
        fl = {n: t[0, h].cpu() for n, t in {**inp, **cot}.items()}
        ref = oracle.attn_jvp_bwd(*(fl[n][None] for n in NAMES), fl["dout"][None], fl["dtout"][None], w.scale,
                                  qrows=rows, krows=keys)
        for n in GRADS:
            sel = rows if n in ("dq", "dtq") else keys
            err[n] = max(err[n], max_rel(got[n][0, h][sel].float().cpu().numpy(), ref[n][0]))
    print(w.name, err)
    for n, e in err.items():
        assert e <= TOL, f"{n}: {e:.3e}"


@pytest.mark.parametrize("H,Lk,parts", [(24, 512, 3), (40, 512, 6), (40, 1024, 4), (40, 2048, 1)])
def test_part_count_on_measured_shapes(H, Lk, parts):
    # the part counts the wave model picks for the key sides of 96, 160, 320 and 640
    # CTAs (32760 queries; 16384 for the first) on a 148-SM B200, each the fastest or
    # within 1 % of it in a sweep of 1..16 parts; read back from the workspace size
    # (statistics, then two regions of parts x heads x keys x 1 KB)
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("part counts measured on 148 SMs")
    Lq = 16384 if H == 24 else 32760
    extra = ajvp.bwd_workspace_bytes(1, H, Lq, Lk) - ajvp.bwd_workspace_bytes(1, H, Lq)
    assert extra == (2 * parts * H * Lk * 1024 if parts > 1 else 0)


def test_split_deterministic_and_close_to_unsplit():
    w = custom(1, 2, 3000, 300, 128)
    inp = gpu_inputs(w, seed=11)
    cot = make_cotangents(w, seed=12, device="cuda")
    a = _bwd(w, inp, cot, split=True)
    b = _bwd(w, inp, cot, split=True)
    c = _bwd(w, inp, cot, split=False)
    for n in GRADS:
        assert torch.equal(a[n], b[n]), n
    # the query side does not split: bit-identical to the unsplit call
    for n in ("dq", "dtq"):
        assert torch.equal(a[n], c[n]), n
    # the key side: the same fp32 sums in another order, rounded to bf16 once
    for n in ("dk", "dv", "dtk", "dtv"):
        x, y = a[n].float(), c[n].float()
        rel = ((x - y).abs().max() / y.abs().max()).item()
        assert rel <= 8e-3, (n, rel)


def test_split_steps_one_at_a_time():
    # attn_jvp_bwd_step runs each kernel on its own; the split steps each end with
    # their reduction, so a step-by-step call equals the whole call
    w = custom(1, 2, 3000, 300, 128)
    inp = gpu_inputs(w, seed=13)
    cot = make_cotangents(w, seed=14, device="cuda")
    whole = _bwd(w, inp, cot, split=True)
    o, to, lse, mu = ajvp.attn_jvp_fwd_stats(*(inp[n] for n in NAMES), w.scale)
    ws = torch.empty(ajvp.bwd_workspace_bytes(w.B, w.H, w.Lq, w.Lk), dtype=torch.uint8, device="cuda")
    grads = {n: torch.full_like(inp["q"] if n in ("dq", "dtq") else inp["k"], 3.0) for n in GRADS}
    for step in range(4):
        ajvp.attn_jvp_bwd(*(inp[n] for n in NAMES), o, to, lse, mu, cot["dout"], cot["dtout"], w.scale,
                          workspace=ws, grads=grads, step=step)
    torch.cuda.synchronize()
    for n in GRADS:
        assert torch.equal(grads[n], whole[n]), n


def test_split_key_steps_on_two_streams():
    # steps 2 (dk, dtk) and 3 (dv, dtv) keep their partial sums in separate regions
    # of the workspace, so they may run at the same time on two streams
    w = custom(1, 2, 3000, 300, 128)
    inp = gpu_inputs(w, seed=18)
    cot = make_cotangents(w, seed=19, device="cuda")
    whole = _bwd(w, inp, cot, split=True)
    o, to, lse, mu = ajvp.attn_jvp_fwd_stats(*(inp[n] for n in NAMES), w.scale)
    ws = torch.empty(ajvp.bwd_workspace_bytes(w.B, w.H, w.Lq, w.Lk), dtype=torch.uint8, device="cuda")
    grads = {n: torch.empty_like(inp["q"] if n in ("dq", "dtq") else inp["k"]) for n in GRADS}
    args = [inp[n] for n in NAMES] + [o, to, lse, mu, cot["dout"], cot["dtout"], w.scale]
    for _ in range(3):
        ajvp.attn_jvp_bwd(*args, workspace=ws, grads=grads, step=0)
        s2, s3 = torch.cuda.Stream(), torch.cuda.Stream()
        s2.wait_stream(torch.cuda.current_stream())
        s3.wait_stream(torch.cuda.current_stream())
        ajvp.attn_jvp_bwd(*args, workspace=ws, grads=grads, step=2, stream=s2)
        ajvp.attn_jvp_bwd(*args, workspace=ws, grads=grads, step=3, stream=s3)
        ajvp.attn_jvp_bwd(*args, workspace=ws, grads=grads, step=1)
        torch.cuda.synchronize()
        for n in GRADS:
            assert torch.equal(grads[n], whole[n]), n
    assert ajvp.check_device_status() == ajvp.AJVP_OK


def test_zero_cotangents_give_zero_gradients():
    w = custom(1, 2, 3000, 300, 128)
    inp = gpu_inputs(w, seed=15)
    zero = {n: torch.zeros_like(inp["q"]) for n in ("dout", "dtout")}
    g = _bwd(w, inp, zero, split=True)
    for n in GRADS:
        assert torch.count_nonzero(g[n]).item() == 0, n


def test_crossattn_workload_sampled():
    # the video cross-attention configuration (B=1, H=40, 32760 queries, 512 keys):
    # the key side splits (160 key tiles); dK..dtV of sampled keys need every query
    # row, dQ and dtQ of sampled rows only their own row
    w = WORKLOADS["video_crossattn_b1h40_lq32760_lk512_d128"]
    assert ajvp.bwd_workspace_bytes(w.B, w.H, w.Lq, w.Lk) > ajvp.bwd_workspace_bytes(w.B, w.H, w.Lq)
    inp = gpu_inputs(w)
    cot = make_cotangents(w, device="cuda")
    got = _bwd(w, inp, cot, split=True)
    rows = sample_rows(w.Lq, 8)
    keys = sample_rows(w.Lk, 10, seed=1)
    err = {n: 0.0 for n in GRADS}
    for h in (0, 17, w.B * w.H - 1):
        fl = {n: t.reshape(-1, t.shape[-2], t.shape[-1])[h].cpu() for n, t in {**inp, **cot}.items()}
        ref = oracle.attn_jvp_bwd(*(fl[n][None] for n in NAMES), fl["dout"][None], fl["dtout"][None], w.scale,
                                  qrows=rows, krows=keys)
        for n in GRADS:
            sel = rows if n in ("dq", "dtq") else keys
            L = w.Lq if n in ("dq", "dtq") else w.Lk
            g = got[n].reshape(-1, L, w.d)[h][sel].float().cpu().numpy()
            err[n] = max(err[n], max_rel(g, ref[n][0]))
    print(w.name, err)
    for n, e in err.items():
        assert e <= TOL, f"{n}: {e:.3e}"
    del inp, cot, got
    torch.cuda.empty_cache()
