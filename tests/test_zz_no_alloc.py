"""attn_jvp_fwd_host_noalloc (host buffers staged through the library's
static 64 MiB device scratch, no allocation in the call) against the
existing host entry point attn_jvp_fwd_host with a caller workspace: two
calls in a row on different inputs must each give bit-identical outputs (the
same kernel on the same slabs; the second call reuses the scratch the first
one filled).  Kept in a file collected last so that it also runs after every
other test in the process; it passes alone as well.  On the CPU: sizes
beyond the scratch are rejected before any CUDA call, and the source of the
entry point and of the pipeline routine it enqueues through creates no
stream or event and allocates nothing outside its one-time per-device set-up
(some callers cannot allocate device memory or create CUDA objects per
call: a plain C caller without a device allocator of its own, or a process
whose device memory a framework's caching allocator already holds)."""
import ctypes
import os
import re

import pytest
import torch

import attention_forward_mode_b200 as ajvp
from attention_forward_mode_b200 import _binding as B
from attention_forward_mode_b200 import build as build_mod
from attention_forward_mode_b200.workloads import custom, make_inputs

NAMES = ("q", "k", "v", "tq", "tk", "tv")
SCRATCH = 64 << 20


def _host_inputs(w, seed):
    return {n: t.pin_memory() for n, t in make_inputs(w, seed=seed, device="cpu").items()}


def _outputs(w):
    shp = (w.B, w.H, w.Lq, w.d)
    return (torch.empty(shp, dtype=torch.bfloat16).pin_memory(), torch.empty(shp, dtype=torch.bfloat16).pin_memory(),
            torch.empty((w.B, w.H, w.Lq), dtype=torch.float32).pin_memory())


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [(2, 3, 1000, 1500), (1, 5, 4096, 4096), (1, 2, 10900, 10900)])
def test_noalloc_equals_host_entry_two_calls(shape):
    w = custom(*shape, 128)
    assert ajvp.host_workspace_bytes(w.Lq, w.Lk, w.d, 1) <= SCRATCH
    ws = torch.empty(ajvp.host_workspace_bytes(w.Lq, w.Lk, w.d, 1), dtype=torch.uint8, device="cuda")
    for seed in (31, 32):  # two calls in a row
        h = _host_inputs(w, seed)
        o, to, lse = _outputs(w)
        ajvp.attn_jvp_fwd_host_noalloc(*(h[n] for n in NAMES), w.scale, o=o, to=to, lse=lse)
        torch.cuda.synchronize()
        ro, rto, rlse = ajvp.attn_jvp_fwd_host(*(h[n] for n in NAMES), w.scale, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(o, ro), ("o", seed)
        assert torch.equal(to, rto), ("to", seed)
        assert torch.equal(lse, rlse), ("lse", seed)


def test_noalloc_rejects_sizes_beyond_the_scratch():
    # host-side check, before any CUDA call: one slab in three buffers > 64 MiB
    build_mod.build()
    lib = B.load_library()
    assert lib.attn_jvp_host_workspace_bytes(10900, 10900, 128, 1) <= SCRATCH
    assert lib.attn_jvp_host_workspace_bytes(10920, 10920, 128, 1) > SCRATCH
    p = ctypes.c_void_p(16)
    rc = lib.attn_jvp_fwd_host_noalloc(p, p, p, p, p, p, p, p, None, 1, 1, 10920, 10920, 128, 0.1, None)
    assert rc == B.AJVP_ERR_TOO_LARGE
    rc = lib.attn_jvp_fwd_host_noalloc(p, p, p, p, p, p, p, p, None, 1, 1, 100, 40000, 128, 0.1, None)
    assert rc == B.AJVP_ERR_TOO_LARGE
    assert lib.attn_jvp_fwd_host_noalloc(p, p, p, p, p, p, p, p, None, 1, 1, 8, 8, 64, 0.1, None) == \
        B.AJVP_ERR_UNSUPPORTED_DIM


def _function_body(src, signature_start):
    """Text of the C function whose definition starts with `signature_start`."""
    i = src.index(signature_start)
    j = src.index("{", i)
    depth = 0
    for k in range(j, len(src)):
        depth += {"{": 1, "}": -1}.get(src[k], 0)
        if depth == 0:
            return src[j:k + 1]
    raise AssertionError("unbalanced braces")


def test_noalloc_path_creates_nothing_per_call():
    # the entry point and the pipeline it enqueues through: the only creation is
    # the one-time set-up inside std::call_once; nothing is freed or destroyed
    src = open(os.path.join(os.path.dirname(B.__file__), "csrc", "api.cu")).read()
    entry = _function_body(src, 'extern "C" int attn_jvp_fwd_host_noalloc(')
    enqueue = _function_body(src, "int fwd_host_enqueue(")
    once = _function_body(entry, "std::call_once(")
    creating = re.compile(r"cuda(Malloc\w*|Free\w*|Stream(Create|Destroy)\w*|Event(Create|Destroy)\w*)\s*\("
                          r"|HostPipe|\.create\(")
    assert creating.search(enqueue) is None, creating.search(enqueue)
    outside = entry.replace(once, "")
    assert creating.search(outside) is None, creating.search(outside)
    assert "pipe.create()" in once and "cudaGetSymbolAddress" in once
