"""CUDA path vs the fp64 oracle on the five named workloads, through the C
ABI, in the launch configuration the benchmark times.  Bounds (max|err| /
max|ref|): bf16 I/O O <= 1e-2, tO <= 2e-2; fp32 I/O <= 1e-4 for both.

Small workloads are checked on every output element.  The full-size video
workloads launch at full size and are checked on sampled query rows of
sampled heads (first, last and one in between); the rows always include
both sides of the first 128-row tile boundaries and the ragged tail.
"""
import pytest
import torch

from attention_forward_mode_b200.workloads import WORKLOADS, custom
from gpu_common import assert_within, compare_full, compare_rows, gpu_inputs, run_cuda

pytestmark = pytest.mark.gpu


def _heads(w):
    bh = w.B * w.H
    return sorted({0, bh // 2, bh - 1})


def test_small_fp32_selfattention_full():
    w = WORKLOADS["selfattn_f32_b1h2_l128_d64"]
    inp = gpu_inputs(w)
    err = compare_full(w, inp, run_cuda(inp, w.scale))
    print(w.name, err)
    assert_within(err, "f32", w.name)


def test_multi_tile_bf16_full():
    """Every element of a case that spans several query tiles and key tiles
    with ragged tails on both (700 = 5 x 128 + 60 = 10 x 64 + 60)."""
    w = custom(1, 3, 700, 700, 128)
    inp = gpu_inputs(w, seed=5)
    err = compare_full(w, inp, run_cuda(inp, w.scale))
    print(w.name, err)
    assert_within(err, "bf16", w.name)


def test_image_selfattention_sampled():
    w = WORKLOADS["image_selfattn_b2h12_l4096_d128"]
    inp = gpu_inputs(w)
    err = compare_rows(w, inp, run_cuda(inp, w.scale), _heads(w), 64)
    print(w.name, err)
    assert_within(err, "bf16", w.name)


def test_video_selfattention_sampled():
    w = WORKLOADS["video_selfattn_b1h12_l32760_d128"]
    inp = gpu_inputs(w)
    err = compare_rows(w, inp, run_cuda(inp, w.scale), _heads(w), 40)
    print(w.name, err)
    assert_within(err, "bf16", w.name)


def test_video_crossattention_sampled():
    w = WORKLOADS["video_crossattn_b1h40_lq32760_lk512_d128"]
    inp = gpu_inputs(w)
    err = compare_rows(w, inp, run_cuda(inp, w.scale), _heads(w) + [7, 23], 256)
    print(w.name, err)
    assert_within(err, "bf16", w.name)


def _widest_score_rows(q, k, n, chunk=4096):
    """The n query rows of one head whose scores q_i . k_j spread widest
    (max_j - min_j, from a bf16 Q K^T on the GPU, in row chunks): the
    peakiest softmax rows, where the lazy rescale and the bf16 rounding of P
    are stressed most."""
    spread = torch.empty(q.shape[0], device=q.device, dtype=torch.float32)
    for r0 in range(0, q.shape[0], chunk):
        s = (q[r0:r0 + chunk] @ k.T).float()
        spread[r0:r0 + chunk] = s.amax(dim=1) - s.amin(dim=1)
        del s
    return sorted(torch.topk(spread, n).indices.tolist())


def test_video_large_selfattention_sampled():
    """Q, K ~ N(0, 2^2): 256 sampled rows on each of three heads, plus the 32
    rows of head 0 with the widest score spread."""
    w = WORKLOADS["video_selfattn_large_b1h40_l75600_d128"]
    inp = gpu_inputs(w)
    out = run_cuda(inp, w.scale)
    err = compare_rows(w, inp, out, _heads(w), 256)
    print(w.name, err)
    assert_within(err, "bf16", w.name)
    wide = _widest_score_rows(inp["q"][0, 0], inp["k"][0, 0], 32)
    err = compare_rows(w, inp, out, [0], 0, rows=wide)
    print(w.name, "widest-spread rows of head 0", wide[:8], err)
    assert_within(err, "bf16", w.name + " (widest-spread rows)")
    del inp, out
    torch.cuda.empty_cache()
