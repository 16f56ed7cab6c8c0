"""The seeded input recipe on the CPU: the documented draw order, the stated
standard deviations and per-key factors, bf16 rounding, and the workload
table's shapes."""
import math

import torch

from attention_forward_mode_b200.workloads import WORKLOADS, custom, make_cotangents, make_inputs

NAMES = ("q", "k", "v", "tq", "tk", "tv")


def test_draw_order_and_rounding():
    # one generator seeded with `seed`: standard normals for Q, K, V, tQ, tK, tV in that
    # order, then the per-key factors uK, uV = U(0,1) * 1.5 + 0.5; rounded to bf16 last
    w = custom(1, 2, 5, 7, 16, kv_row_scale=True, t_std=0.25)
    got = make_inputs(w, seed=9)
    g = torch.Generator().manual_seed(9)
    shp = {"q": (1, 2, 5, 16), "tq": (1, 2, 5, 16)}
    raw = {n: torch.randn(shp.get(n, (1, 2, 7, 16)), generator=g) for n in NAMES}
    uk = torch.rand((1, 2, 7), generator=g) * 1.5 + 0.5
    uv = torch.rand((1, 2, 7), generator=g) * 1.5 + 0.5
    ref = {"q": raw["q"], "k": raw["k"] * uk[..., None], "v": raw["v"] * uv[..., None],
           "tq": raw["tq"] * 0.25, "tk": raw["tk"] * 0.25, "tv": raw["tv"] * 0.25}
    for n in NAMES:
        assert got[n].dtype == torch.bfloat16 and got[n].is_contiguous()
        assert torch.equal(got[n], ref[n].to(torch.bfloat16)), n


def test_seeds():
    w = custom(1, 1, 33, 17, 128)
    a, b, c = make_inputs(w, seed=1), make_inputs(w, seed=1), make_inputs(w, seed=2)
    for n in NAMES:
        assert torch.equal(a[n], b[n]) and not torch.equal(a[n], c[n]), n
    d1, d2 = make_cotangents(w, seed=1), make_cotangents(w, seed=1)
    assert torch.equal(d1["dout"], d2["dout"]) and not torch.equal(d1["dout"], d1["dtout"])
    assert d1["dout"].shape == (1, 1, 33, 128) and d1["dtout"].dtype == torch.bfloat16


def test_stated_spreads():
    # sample standard deviations of the stated distributions (about 1 % noise at these sizes)
    w = custom(1, 4, 4096, 4096, 128, q_std=2.0, k_std=2.0, t_std=0.1)
    x = make_inputs(w, seed=3)
    for n, s in (("q", 2.0), ("k", 2.0), ("v", 1.0), ("tq", 0.1), ("tk", 0.1), ("tv", 0.1)):
        sd = x[n].float().std().item()
        assert abs(sd / s - 1.0) < 0.02, (n, sd)
        assert abs(x[n].float().mean().item()) < 0.02 * s, n


def test_per_key_factors_span_half_to_two():
    w = custom(1, 2, 8, 4096, 128, kv_row_scale=True)
    x = make_inputs(w, seed=4)
    for n in ("k", "v"):
        rms = x[n].float().pow(2).mean(-1).sqrt()          # per key: |U| x (chi / sqrt(128))
        assert 0.35 < rms.min().item() < 0.6 and 1.8 < rms.max().item() < 2.6, n
        # U(0.5, 2) has mean 1.25; E[chi_128 / sqrt(128)] is within 0.2 % of 1
        assert abs(rms.mean().item() / 1.25 - 1.0) < 0.03, n
    for n in ("q", "tq", "tk", "tv"):
        rms = x[n].float().pow(2).mean(-1).sqrt()
        assert rms.max().item() < 1.3, n


def test_workload_table():
    shapes = {n: (w.B, w.H, w.Lq, w.Lk, w.d, w.dtype) for n, w in WORKLOADS.items()}
    assert shapes["selfattn_f32_b1h2_l128_d64"] == (1, 2, 128, 128, 64, "f32")
    assert shapes["image_selfattn_b2h12_l4096_d128"] == (2, 12, 64 * 64, 64 * 64, 128, "bf16")
    assert shapes["video_selfattn_b1h12_l32760_d128"] == (1, 12, 21 * 30 * 52, 21 * 30 * 52, 128, "bf16")
    assert shapes["video_crossattn_b1h40_lq32760_lk512_d128"] == (1, 40, 21 * 30 * 52, 512, 128, "bf16")
    assert shapes["video_selfattn_large_b1h40_l75600_d128"] == (1, 40, 21 * 45 * 80, 21 * 45 * 80, 128, "bf16")
    for w in WORKLOADS.values():
        assert math.isclose(w.scale, 1.0 / math.sqrt(w.d))
        assert w.flops == 12 * w.B * w.H * w.Lq * w.Lk * w.d
