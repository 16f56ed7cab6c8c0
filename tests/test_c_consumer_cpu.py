"""The boundary from a plain C99 program: it includes include/attn_jvp.h,
links libattnjvp.so with gcc and calls the host-side queries and argument
checks (no GPU needed), as a C caller with no Python or torch would."""
import os
import shutil
import subprocess

import pytest

from attention_forward_mode_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "attn_jvp.h"

int main(void) {
    int bad = 0;
    /* size queries: plain host arithmetic */
    if (attn_jvp_bwd_workspace_bytes(1, 2, 100) != 4352u) bad |= 1;
    if (attn_jvp_bwd_key_split_parts(1, 40, 32760, 512, 148) != 6) bad |= 2;
    if (attn_jvp_bwd_key_split_parts(1, 40, 32760, 2048, 148) != 1) bad |= 4;
    if (attn_jvp_host_workspace_bytes(0, 8, 128, 1) != 0u) bad |= 8;
    /* host-side argument checks return before any CUDA call */
    char buf[64];
    void *p = buf + (16 - ((size_t)buf & 15));  /* 16-byte aligned, never dereferenced */
    if (attn_jvp_fwd(NULL, p, p, p, p, p, p, p, NULL, 1, 1, 8, 8, 128, 0.1f, NULL) != AJVP_ERR_INVALID_ARG)
        bad |= 16;
    if (attn_jvp_fwd(p, p, p, p, p, p, p, p, NULL, 1, 1, 8, 0, 128, 0.1f, NULL) != AJVP_ERR_INVALID_ARG)
        bad |= 32;
    if (attn_jvp_fwd(p, p, p, p, p, p, p, p, NULL, 0, 1, 8, 8, 128, 0.1f, NULL) != AJVP_OK) bad |= 64;
    const char *msg = attn_jvp_strerror(AJVP_ERR_INVALID_ARG);
    if (!msg || !strlen(msg)) bad |= 128;
    printf("bad=%d\n", bad);
    return bad != 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c99_program_links_and_calls(tmp_path):
    lib = build_mod.build()
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-L", libdir, "-lattnjvp", "-Wl,-rpath," + libdir, "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and "bad=0" in r.stdout, (r.stdout, r.stderr)
