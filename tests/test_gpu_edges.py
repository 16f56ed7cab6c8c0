"""Edge cases of the CUDA path against the fp64 oracle and the method's
invariants: ragged and tiny shapes, Lq != Lk both ways, more heads than SMs,
empty inputs, zero and degenerate tangents, odd scales, the failure-detection
self test."""
import pytest
import torch

import attention_forward_mode_b200 as ajvp
from attention_forward_mode_b200.workloads import custom, make_inputs
from gpu_common import assert_within, compare_full, gpu_inputs, max_rel, run_cuda

pytestmark = pytest.mark.gpu

BF16_SHAPES = [  # (B, H, Lq, Lk)
    (1, 1, 1, 1), (1, 1, 1, 200), (1, 2, 5, 64), (1, 1, 63, 65), (1, 2, 128, 128),
    (1, 1, 129, 127), (1, 2, 200, 1), (1, 1, 256, 3), (2, 3, 300, 2000), (1, 1, 257, 4097),
    (1, 2, 1000, 130),
]


@pytest.mark.parametrize("B,H,Lq,Lk", BF16_SHAPES)
def test_bf16_shapes(B, H, Lq, Lk):
    w = custom(B, H, Lq, Lk, 128)
    inp = gpu_inputs(w, seed=Lq * 7 + Lk)
    err = compare_full(w, inp, run_cuda(inp, w.scale))
    assert_within(err, "bf16", w.name)


F32_SHAPES = [  # (B, H, Lq, Lk, d)
    (1, 1, 1, 1, 64), (1, 2, 17, 33, 64), (2, 1, 100, 70, 128), (1, 1, 40, 300, 256),
    (1, 3, 65, 31, 32), (1, 1, 33, 47, 100), (1, 1, 8, 9, 1),
]


@pytest.mark.parametrize("B,H,Lq,Lk,d", F32_SHAPES)
def test_f32_shapes(B, H, Lq, Lk, d):
    w = custom(B, H, Lq, Lk, d, dtype="f32")
    inp = gpu_inputs(w, seed=d + Lq)
    err = compare_full(w, inp, run_cuda(inp, w.scale))
    assert_within(err, "f32", w.name)


def test_more_heads_than_sms():
    w = custom(3, 60, 130, 70, 128)  # 180 heads x 2 query tiles
    inp = gpu_inputs(w, seed=3)
    err = compare_full(w, inp, run_cuda(inp, w.scale))
    assert_within(err, "bf16", w.name)


@pytest.mark.parametrize("scale", [-0.2, 0.0, 0.5])
def test_unusual_scales(scale):
    w = custom(1, 2, 150, 190, 128, scale=scale)
    inp = gpu_inputs(w, seed=9)
    err = compare_full(w, inp, run_cuda(inp, w.scale))
    assert_within(err, "bf16", w.name)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_zero_tangent_gives_exact_zero(dtype):
    w = custom(1, 2, 300, 260, 128 if dtype == "bf16" else 64, dtype=dtype)
    inp = gpu_inputs(w, seed=1)
    for n in ("tq", "tk", "tv"):
        inp[n].zero_()
    _, to, _ = run_cuda(inp, w.scale)
    assert torch.count_nonzero(to).item() == 0


def test_shift_invariance():
    """tQ = 0, tK = one vector c for every key, tV = 0: each row's scores move
    by the same amount, softmax does not change, tO = 0 up to rounding."""
    w = custom(1, 2, 256, 400, 128)
    inp = gpu_inputs(w, seed=2)
    inp["tq"].zero_()
    inp["tv"].zero_()
    c = torch.randn(1, 2, 1, 128, device="cuda").to(torch.bfloat16)
    inp["tk"].copy_(c.expand_as(inp["tk"]))
    o, to, _ = run_cuda(inp, w.scale)
    shift = (inp["q"].float() @ c.float().transpose(-1, -2)).abs().max().item() * w.scale
    bound = 1e-2 * shift * inp["v"].float().abs().max().item()
    assert to.float().abs().max().item() <= bound


def test_ptv_term_equals_attention_of_tv():
    """tQ = tK = 0: tO must equal attention(Q, K, tV), i.e. the kernel's own
    O with V replaced by tV."""
    w = custom(1, 2, 333, 500, 128)
    inp = gpu_inputs(w, seed=4)
    inp["tq"].zero_()
    inp["tk"].zero_()
    _, to, _ = run_cuda(inp, w.scale)
    inp2 = dict(inp)
    inp2["v"] = inp["tv"].clone()
    o2, _, _ = run_cuda(inp2, w.scale)
    assert max_rel(to.float().cpu().numpy(), o2.float().cpu().numpy()) <= 1e-2


def test_empty_inputs_are_noops():
    w = custom(1, 2, 0, 64, 128)
    inp = make_inputs(w, device="cuda")
    o = torch.full((1, 2, 0, 128), 1.0, device="cuda", dtype=torch.bfloat16)
    out = ajvp.attn_jvp_fwd(inp["q"], inp["k"], inp["v"], inp["tq"], inp["tk"], inp["tv"], 0.1, o=o)
    torch.cuda.synchronize()
    assert out[0].numel() == 0


def test_lse_optional_and_outputs_identical():
    w = custom(1, 2, 200, 300, 128)
    inp = gpu_inputs(w, seed=6)
    a = ajvp.attn_jvp_fwd(inp["q"], inp["k"], inp["v"], inp["tq"], inp["tk"], inp["tv"], w.scale)
    b = ajvp.attn_jvp_fwd(inp["q"], inp["k"], inp["v"], inp["tq"], inp["tk"], inp["tv"], w.scale,
                          want_lse=False)
    torch.cuda.synchronize()
    assert b[2] is None
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_deterministic_and_side_stream():
    w = custom(2, 2, 260, 700, 128)
    inp = gpu_inputs(w, seed=8)
    a = run_cuda(inp, w.scale)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = ajvp.attn_jvp_fwd(inp["q"], inp["k"], inp["v"], inp["tq"], inp["tk"], inp["tv"], w.scale, stream=s)
    s.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bad_arguments_raise():
    w = custom(1, 1, 16, 16, 64)
    inp = make_inputs(w, device="cuda")  # d = 64 is not supported by the bf16 kernel
    with pytest.raises(ajvp.AttnJvpError) as e:
        ajvp.attn_jvp_fwd(inp["q"], inp["k"], inp["v"], inp["tq"], inp["tk"], inp["tv"])
    assert e.value.status == ajvp.AJVP_ERR_UNSUPPORTED_DIM


def test_wait_timeout_is_detected_and_context_survives():
    """A bounded wait on a barrier nothing completes gives up after ~1 ms,
    the device status word reports it, and the next launch works."""
    assert ajvp.check_device_status() == ajvp.AJVP_OK
    ajvp.selftest_wait_timeout(1_000_000)
    assert ajvp.check_device_status() == ajvp.AJVP_ERR_TIMEOUT
    assert ajvp.check_device_status() == ajvp.AJVP_OK  # read-and-clear
    w = custom(1, 1, 130, 70, 128)
    inp = gpu_inputs(w, seed=1)
    err = compare_full(w, inp, run_cuda(inp, w.scale))
    assert_within(err, "bf16", w.name)
    assert ajvp.check_device_status() == ajvp.AJVP_OK
