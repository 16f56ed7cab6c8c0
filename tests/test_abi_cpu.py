"""C ABI checks that need no GPU: the library loads, exports every symbol
the header declares, and rejects bad arguments on the host before touching
CUDA."""
import ctypes
import os
import re

import pytest

from attention_forward_mode_b200 import _binding as B
from attention_forward_mode_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.load_library()


def header_functions():
    text = open(os.path.join(ROOT, "include", "attn_jvp.h")).read()
    return sorted(set(re.findall(r"AJVP_API\s+[\w\s\*]*?\b(attn_jvp_\w+)\s*\(", text)))


def test_header_matches_binding_list():
    assert header_functions() == sorted(B.EXPORTED)


def test_every_header_symbol_exported(lib):
    raw = ctypes.CDLL(B.LIB_PATH)
    for name in header_functions():
        assert hasattr(raw, name), name


def test_version_and_strerror(lib):
    assert lib.attn_jvp_version() == 100
    for code in range(-9, 1):
        assert len(lib.attn_jvp_strerror(code)) > 5
    assert b"unknown" in lib.attn_jvp_strerror(-99)


def _call(lib, fn="attn_jvp_fwd", ptr=16, B_=1, H=1, Lq=8, Lk=8, d=128, scale=0.1, lse=None):
    f = getattr(lib, fn)
    p = ctypes.c_void_p(ptr) if ptr is not None else None
    return f(p, p, p, p, p, p, p, p, lse, B_, H, Lq, Lk, d, scale, None)


@pytest.mark.parametrize("fn", ["attn_jvp_fwd", "attn_jvp_fwd_f32"])
def test_host_side_rejections(lib, fn):
    # none of these reach a CUDA call: checked on the host first
    assert _call(lib, fn, Lk=0) == B.AJVP_ERR_INVALID_ARG
    assert _call(lib, fn, Lq=-1) == B.AJVP_ERR_INVALID_ARG
    assert _call(lib, fn, B_=-2) == B.AJVP_ERR_INVALID_ARG
    assert _call(lib, fn, d=0) == B.AJVP_ERR_INVALID_ARG
    assert _call(lib, fn, scale=float("nan")) == B.AJVP_ERR_INVALID_ARG
    assert _call(lib, fn, scale=float("inf")) == B.AJVP_ERR_INVALID_ARG
    assert _call(lib, fn, ptr=None) == B.AJVP_ERR_INVALID_ARG
    assert _call(lib, fn, Lq=1 << 31) == B.AJVP_ERR_TOO_LARGE
    assert _call(lib, fn, Lk=1 << 31) == B.AJVP_ERR_TOO_LARGE
    # empty work is a successful no-op (null pointers allowed then)
    assert _call(lib, fn, ptr=None, Lq=0) == B.AJVP_OK
    assert _call(lib, fn, ptr=None, B_=0) == B.AJVP_OK
    assert _call(lib, fn, ptr=None, H=0) == B.AJVP_OK


def test_bf16_dim_and_alignment_rules(lib):
    assert _call(lib, d=64) == B.AJVP_ERR_UNSUPPORTED_DIM
    assert _call(lib, d=256) == B.AJVP_ERR_UNSUPPORTED_DIM
    assert _call(lib, ptr=24) == B.AJVP_ERR_MISALIGNED
    assert _call(lib, lse=ctypes.c_void_p(20)) == B.AJVP_ERR_MISALIGNED


def _call_host(lib, ptr=16, Lq=8, Lk=8, d=128, ws=256, ws_bytes=None):
    p = ctypes.c_void_p(ptr) if ptr is not None else None
    w = ctypes.c_void_p(ws) if ws is not None else None
    if ws_bytes is None:
        ws_bytes = lib.attn_jvp_host_workspace_bytes(Lq, Lk, d, 1)
    return lib.attn_jvp_fwd_host(p, p, p, p, p, p, p, p, None, 1, 1, Lq, Lk, d, 0.1, w, ws_bytes, None)


def test_host_workspace_bytes(lib):
    f = lib.attn_jvp_host_workspace_bytes
    assert f(0, 8, 128, 1) == 0 and f(8, 8, 128, 0) == 0
    # three buffers; per buffer 2 q-side + 4 k-side inputs, 2 outputs, lse, each rounded to 256 bytes
    per = 4 * 8 * 128 * 2 + 4 * 16 * 128 * 2 + 256
    assert f(8, 16, 128, 1) == 3 * per
    assert f(8, 16, 128, 3) == 3 * (4 * 3 * 8 * 128 * 2 + 4 * 3 * 16 * 128 * 2 + 256)
    assert f(1, 1, 128, 1) == 3 * 9 * 256  # every array padded to its own 256-byte boundary


def test_bwd_workspace_bytes(lib):
    f, fs = lib.attn_jvp_bwd_workspace_bytes, lib.attn_jvp_bwd_workspace_bytes_split
    # per (batch, head) row 16 bytes of statistics, 64 rows of padding, rounded to 256
    assert f(1, 2, 100) == 4352  # (200 + 64) x 16 = 4224, rounded up
    assert f(2, 3, 4096) == (6 * 4096 + 64) * 16
    assert f(-1, 2, 100) == 0 and fs(1, 2, 100, -1) == 0
    # no usable device here: the split size is the minimum (the kernels then do not split)
    for shape in ((1, 40, 32760, 512), (1, 2, 3000, 300), (1, 12, 32760, 32760)):
        assert fs(*shape) == f(*shape[:3]), shape


def test_bwd_key_split_parts(lib):
    f = lib.attn_jvp_bwd_key_split_parts
    # the counts a sweep of 1..16 parts measured fastest (or within 1 %) on a 148-SM B200:
    # key sides of 96, 160, 320 and 640 CTAs
    assert f(1, 24, 16384, 512, 148) == 3
    assert f(1, 40, 32760, 512, 148) == 6
    assert f(1, 40, 32760, 1024, 148) == 4
    assert f(1, 40, 32760, 2048, 148) == 1
    # invalid arguments
    assert f(-1, 1, 64, 64, 148) == 0 and f(1, 1, 64, 64, 0) == 0 and f(1, 1, 64, -1, 148) == 0
    # properties over a grid of shapes: 1 <= parts <= min(16, query tiles); no split when the
    # key tiles give four CTAs per SM or there is one query tile; no part is empty
    for sm in (148, 132, 8):
        for bh in (1, 3, 24, 40, 200):
            for Lq in (1, 64, 65, 1000, 4100, 32760):
                for Lk in (1, 77, 512, 1024, 4096):
                    s = f(1, bh, Lq, Lk, sm)
                    tiles, ctas = -(-Lq // 64), -(-Lk // 128) * bh
                    assert 1 <= s <= max(1, min(16, tiles)), (sm, bh, Lq, Lk, s)
                    if ctas >= 4 * sm or tiles <= 1:
                        assert s == 1, (sm, bh, Lq, Lk, s)
                    chunk = -(-tiles // s)
                    assert (s - 1) * chunk < tiles, (sm, bh, Lq, Lk, s)
    assert B.bwd_key_split_parts(1, 40, 32760, 512, sm_count=148) == 6


def test_host_entry_rejections(lib):
    # host-side checks, before any CUDA call
    assert _call_host(lib, Lk=0) == B.AJVP_ERR_INVALID_ARG
    assert _call_host(lib, d=64) == B.AJVP_ERR_UNSUPPORTED_DIM
    assert _call_host(lib, ws=None) == B.AJVP_ERR_WORKSPACE
    assert _call_host(lib, ws=128) == B.AJVP_ERR_WORKSPACE  # not 256-byte aligned
    need = lib.attn_jvp_host_workspace_bytes(8, 8, 128, 1)
    assert _call_host(lib, ws_bytes=need - 1) == B.AJVP_ERR_WORKSPACE
    assert _call_host(lib, ptr=None, Lq=0, ws=None) == B.AJVP_OK  # empty: no-op


def test_f32_dim_and_alignment_rules(lib):
    assert _call(lib, "attn_jvp_fwd_f32", d=257) == B.AJVP_ERR_UNSUPPORTED_DIM
    assert _call(lib, "attn_jvp_fwd_f32", ptr=18) == B.AJVP_ERR_MISALIGNED


def test_no_gpu_reports_cuda_or_device_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # valid arguments: the first CUDA call fails on a machine without a GPU
    rc = _call(lib, ptr=1 << 20)
    assert rc in (B.AJVP_ERR_CUDA, B.AJVP_ERR_UNSUPPORTED_DEVICE)


def test_binding_raises_without_cuda_tensors(lib):
    import torch
    x = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        B.attn_jvp_fwd(x, x, x, x, x, x)


def test_varlen_host_rejections(lib):
    f = lib.attn_jvp_fwd_varlen
    vp = ctypes.c_void_p
    p = vp(16)

    def call(cu=vp(64), n_seq=2, total_q=100, total_k=90, max_q=60, d=128):
        return f(p, p, p, p, p, p, p, p, None, cu, cu, n_seq, 2, total_q, total_k, max_q, d, 0.1, 0, None)

    assert call(n_seq=0) == B.AJVP_OK and call(max_q=0) == B.AJVP_OK  # nothing to compute
    assert call(cu=None) == B.AJVP_ERR_INVALID_ARG
    assert call(cu=vp(66)) == B.AJVP_ERR_MISALIGNED
    assert call(max_q=101) == B.AJVP_ERR_INVALID_ARG  # longer than the packed tensor
    assert call(total_k=0) == B.AJVP_ERR_INVALID_ARG
    assert call(d=64) == B.AJVP_ERR_UNSUPPORTED_DIM


def test_persistent_key_tiles_setting(lib):
    """The scheduling knob accepts 0 (off) and positive tile counts, rejects
    negative ones, and needs no GPU."""
    assert lib.attn_jvp_set_persistent_key_tiles(-1) == B.AJVP_ERR_INVALID_ARG
    assert lib.attn_jvp_set_persistent_key_tiles(0) == B.AJVP_OK
    assert lib.attn_jvp_set_persistent_key_tiles(B.DEFAULT_PERSISTENT_KEY_TILES) == B.AJVP_OK


def test_bwd_pairs_setting(lib):
    """The backward's pair switch takes any int (0 off, else on) and needs no GPU."""
    assert lib.attn_jvp_set_bwd_pairs(0) == B.AJVP_OK
    assert lib.attn_jvp_set_bwd_pairs(7) == B.AJVP_OK
    assert lib.attn_jvp_set_bwd_pairs(1) == B.AJVP_OK

