"""The benchmark's reference arm (the fp64 oracle timed on the host cores) on
the CPU: one JSON line with the contract's keys, and under a two-rank
launcher rank 0 alone prints it while the other rank exits 0."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ARGS = ["--impl", "reference", "--workload", "image_selfattn_b2h12_l4096_d128", "--steps", "1", "--warmup", "3",
        "--reference-seconds", "2"]


def _lines(out):
    return [json.loads(s) for s in out.splitlines() if s.startswith("{")]


def _check(line, entry_metric_word):
    assert line["impl"] == "reference" and line["dtype"] == "f64" and line["data"] == "synthetic"
    assert entry_metric_word in line["metric"] and line["unit"] == "TFLOP/s" and line["higher_is_better"]
    assert line["value"] > 0 and line["steps"] == 1 and line["warmup"] >= 3
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "image_selfattn_b2h12_l4096_d128"


@pytest.mark.timeout(300)
@pytest.mark.parametrize("entry,word", [("bf16", "attention+JVP TFLOP/s"), ("bwd", "backward")])
def test_reference_line(entry, word):
    r = subprocess.run([sys.executable, "bench.py", *ARGS, "--entry", entry], cwd=ROOT, capture_output=True,
                       text=True, timeout=280)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _lines(r.stdout)
    assert len(lines) == 1, r.stdout
    _check(lines[0], word)


@pytest.mark.timeout(300)
def test_reference_two_ranks_rank0_prints():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", *ARGS, "--gpus", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=280,
                       env={**os.environ, "OMP_NUM_THREADS": "4"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _lines(r.stdout)
    assert len(lines) == 1, r.stdout
    _check(lines[0], "attention+JVP TFLOP/s")
    assert lines[0]["n_gpus"] == 2
