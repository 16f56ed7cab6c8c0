"""The persistent form of the unmasked bf16 forward (short key sequences,
more query tiles than SMs): every element against the fp64 oracle on cases
where each CTA walks several query tiles with ragged tails on both sides,
and bit-for-bit equality with the one-CTA-per-tile launch of the same call
(the per-tile arithmetic is the same; only the scheduling differs).  Keys
in 3 to 32 tiles of 64 take the persistent form; fewer than 3 run per tile
(the 37-key case checks that the launch still matches)."""
import pytest
import torch

import attention_forward_mode_b200 as ajvp
from attention_forward_mode_b200.workloads import WORKLOADS, custom
from gpu_common import assert_within, compare_full, compare_rows, gpu_inputs, run_cuda

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "tq", "tk", "tv")


def _both(inp, scale, stats=False):
    """(persistent, per-tile) results of the same call."""
    fn = ajvp.attn_jvp_fwd_stats if stats else ajvp.attn_jvp_fwd
    outs = []
    try:
        for tiles in (ajvp.DEFAULT_PERSISTENT_KEY_TILES, 0):
            ajvp.set_persistent_key_tiles(tiles)
            outs.append(fn(*(inp[n] for n in NAMES), scale))
            torch.cuda.synchronize()
    finally:
        ajvp.set_persistent_key_tiles(ajvp.DEFAULT_PERSISTENT_KEY_TILES)
    return outs


@pytest.mark.parametrize("B,H,Lq,Lk", [
    (2, 5, 4000, 200),   # 320 query tiles, 4 key tiles (last one ragged)
    (1, 16, 1500, 150),  # three key tiles (the fewest the persistent form takes), the last ragged
    (3, 7, 900, 700),    # 11 key tiles, 8 ragged query tiles per head
])
def test_persistent_full_against_oracle(B, H, Lq, Lk):
    w = custom(B, H, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=Lq + 3 * Lk)
    err = compare_full(w, inp, run_cuda(inp, w.scale))
    print(w.name, err)
    assert_within(err, "bf16", w.name)


@pytest.mark.parametrize("B,H,Lq,Lk", [(2, 5, 4000, 200), (1, 16, 1500, 150), (1, 16, 1500, 37),
                                        (1, 12, 2000, 2048)])
def test_persistent_bitwise_equals_per_tile_launch(B, H, Lq, Lk):
    w = custom(B, H, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=11)
    a, b = _both(inp, w.scale, stats=True)
    for x, y, name in zip(a, b, ("o", "to", "lse", "mu")):
        assert torch.equal(x, y), name


def test_threshold_edge_against_oracle():
    """2048 keys (32 tiles: persistent) and 2049 (per-tile), sampled rows."""
    for Lk in (2048, 2049):
        w = custom(1, 12, 2000, Lk, 128)
        inp = gpu_inputs(w, seed=Lk)
        err = compare_rows(w, inp, run_cuda(inp, w.scale), [0, 5, 11], 96)
        print(w.name, err)
        assert_within(err, "bf16", w.name)


def test_crossattention_workload_bitwise():
    """The 512-text-key cross-attention workload at full size, both launches."""
    w = WORKLOADS["video_crossattn_b1h40_lq32760_lk512_d128"]
    inp = gpu_inputs(w)
    a, b = _both(inp, w.scale)
    for x, y, name in zip(a, b, ("o", "to", "lse")):
        assert torch.equal(x, y), name
    del inp, a, b
    torch.cuda.empty_cache()
