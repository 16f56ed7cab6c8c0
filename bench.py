"""Benchmark of the fused attention + JVP forward pass on B200.

One step = one call of the C ABI's ``attn_jvp_fwd`` on the whole workload
(the 32760-token video self-attention JVP by default: B=1, H=12,
Lq=Lk=32760, d=128, bf16 I/O).  Metric: attention+JVP TFLOP/s, counting
12 * Lq * Lk * d FLOPs per head, and its fraction of the measured B200 dense
bf16 tensor peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 launch one process per GPU with torch.distributed.run; every rank
runs its own replica of the workload (independent problems, no data-path
collective: weak scaling) and rank 0 prints one JSON line with the job-wide
aggregate over the max-over-ranks device time.

``--impl reference`` times the fp64 CPU oracle (plain loops, OpenMP) on a
bounded sample of the same workload on this machine's host cores: the only
other implementation there is of this computation.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from attention_forward_mode_b200.workloads import BENCH_WORKLOAD, WORKLOADS, make_inputs  # noqa: E402

METRIC = "attention+JVP TFLOP/s (12·Lq·Lk·d/head) and % of B200 BF16 tensor peak"
FALLBACK_BF16_TFLOPS = 1590.0
KERNEL_SOURCES = ["attention_forward_mode_b200/csrc/jvp_sm100.cuh", "attention_forward_mode_b200/csrc/ptx_sm100.cuh"]
TRAFFIC_FILE = "profiles/attn_jvp_fwd_kernel.video_selfattn_b1h12_l32760.md"
# forward workloads with a committed ncu summary of their bf16 kernel (DRAM bytes per launch)
FWD_TRAFFIC_FILES = {"video_selfattn_b1h12_l32760_d128": TRAFFIC_FILE,
                     "video_crossattn_b1h40_lq32760_lk512_d128":
                         "profiles/attn_jvp_fwd_kernel_persistent.video_crossattn_b1h40_lq32760_lk512.md"}
# the same for the fp32-output instantiation (--entry f32out)
F32OUT_TRAFFIC_FILES = {"video_selfattn_b1h12_l32760_d128":
                        "profiles/attn_jvp_fwd_kernel_f32out.video_selfattn_b1h12_l32760.md"}
MASKED_METRIC = "attention+JVP TFLOP/s (12·d per visible query-key pair) and % of B200 BF16 tensor peak"
BWD_METRIC = "attention+JVP backward TFLOP/s (30·Lq·Lk·d/head) and % of B200 BF16 tensor peak"
BWD_MASKED_METRIC = ("attention+JVP masked backward TFLOP/s (30·d per visible query-key pair) and % of B200 "
                     "BF16 tensor peak")
BWD_KERNEL_SOURCES = ["attention_forward_mode_b200/csrc/jvp_bwd_sm100.cuh",
                      "attention_forward_mode_b200/csrc/ptx_sm100.cuh"]
BWD_TRAFFIC_FILE = "profiles/attn_jvp_bwd_kernel.video_selfattn_b1h12_l32760.md"
BWD_TRAFFIC_WORKLOAD = "video_selfattn_b1h12_l32760_d128"  # the workload and kernel (V_K) it covers
L2_BYTES = 126 * 1024 * 1024
# backward kernels (steps of attn_jvp_bwd): name, contraction FLOPs per (Lq*Lk*d) per head
BWD_STEPS = [("bwd_rowstats_kernel", 0.0), ("attn_jvp_bwd_kernel<V_Q> (dQ, dtQ)", 18.0),
             ("attn_jvp_bwd_kernel<V_K> (dK, dtK)", 18.0), ("attn_jvp_bwd_kernel<V_V> (dV, dtV)", 12.0)]


# ------------------------------------------------------------------ helpers
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world: int, local: int, backend: str = "nccl", timeout_s: int = 300):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return dist


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(flops_per_rank_step: float, steps: int, world: int, max_seconds: float) -> float:
    """Whole-job TFLOP/s: every rank's work over the slowest rank's time."""
    return flops_per_rank_step * steps * world / max_seconds / 1e12


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["bf16_tflops"]), float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def kernel_source_sha(sources=None) -> str:
    """Hash of the kernel sources' code: comments and whitespace are dropped, so
    that a comment-only edit does not invalidate a committed ncu capture."""
    h = hashlib.sha256()
    for rel in sources or KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)  # block comments
        text = re.sub(r"//[^\n]*", " ", text)                 # line comments
        h.update("".join(text.split()).encode())
    return h.hexdigest()[:16]


def committed_traffic(traffic_file=TRAFFIC_FILE, sources=None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the kernel source as it stands (else None)."""
    path = os.path.join(ROOT, traffic_file)
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line and line.strip().startswith(("traffic_bytes_per_launch", "kernel_source_sha")):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("kernel_source_sha") != kernel_source_sha(sources):
        return None
    try:
        return float(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling while the timed region runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=self.out,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if getattr(self, "out", None):
            self.out.close()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        mx = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        loaded = [s for s in sm if s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit()) if rows else None}


# ------------------------------------------------------------- CPU oracle
def oracle_sample(w, inputs_cpu_head, seconds: float, seed: int = 0):
    """Time the fp64 oracle on query rows of one head (all Lk keys) for about
    ``seconds``; returns (TFLOP/s-equivalent, rows, elapsed, threads)."""
    import oracle
    q, k, v, tq, tk, tv = inputs_cpu_head
    g = torch.Generator().manual_seed(seed)
    # calibrate on two rows per oracle thread (rows are spread over threads)
    probe = max(4, 2 * oracle.num_threads())
    idx = torch.randperm(q.shape[0], generator=g)[:probe]
    t0 = time.perf_counter()
    oracle.attn_jvp(q[idx][None], k[None], v[None], tq[idx][None], tk[None], tv[None], w.scale)
    per_row = max((time.perf_counter() - t0) / probe, 1e-6)
    rows = int(max(1, min(q.shape[0], seconds / per_row)))
    idx = torch.randperm(q.shape[0], generator=g)[:rows]
    qs, tqs = q[idx][None], tq[idx][None]
    t0 = time.perf_counter()
    oracle.attn_jvp(qs, k[None], v[None], tqs, tk[None], tv[None], w.scale)
    el = time.perf_counter() - t0
    flops = 12.0 * rows * w.Lk * w.d
    return flops / el / 1e12, rows, el, oracle.num_threads()


def causal_flops(w) -> float:
    """12 d FLOPs per visible (query, key) pair of the causal mask (key j
    visible to query i iff j <= i + Lk - Lq), summed over the heads."""
    i = torch.arange(w.Lq, dtype=torch.float64)
    vis = torch.clamp(i + (w.Lk - w.Lq) + 1, 0, w.Lk).sum().item()
    return 12.0 * w.d * w.B * w.H * vis


def oracle_sample_causal(w, inputs_cpu_head, seconds: float):
    """Time the fp64 masked oracle on the causal sub-problem made of the first
    n query rows and the first n + Lk - Lq keys of one head (complete, so its
    FLOPs are those of an n-row causal problem), n sized to about ``seconds``."""
    import oracle
    q, k, v, tq, tk, tv = inputs_cpu_head
    off = w.Lk - w.Lq

    def run(n):
        nk = max(1, min(w.Lk, n + off))
        t0 = time.perf_counter()
        oracle.attn_jvp_causal(q[:n][None], k[:nk][None], v[:nk][None], tq[:n][None], tk[:nk][None],
                               tv[:nk][None], w.scale)
        el = time.perf_counter() - t0
        i = torch.arange(n, dtype=torch.float64)
        vis = torch.clamp(i + (nk - n) + 1, 0, nk).sum().item()
        return el, 12.0 * w.d * vis

    n0 = min(w.Lq, 512)
    el0, _ = run(n0)
    n = int(min(w.Lq, max(n0, n0 * (seconds / max(el0, 1e-6)) ** 0.5)))
    el, fl = run(n)
    return fl / el / 1e12, n, el, oracle.num_threads()


def head0_cpu(inp):
    return tuple(inp[n][0, 0].detach().cpu() for n in ("q", "k", "v", "tq", "tk", "tv"))


# ------------------------------------------------------------------ arms
def run_reference(args, w):
    rank, world, local = dist_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    inp = make_inputs(w, seed=0, device="cpu")
    head = head0_cpu(inp)
    del inp
    total_steps = args.steps + args.warmup
    per_step = max(0.5, args.reference_seconds / max(1, total_steps))
    # bounded sample per step: rows of head 0 sized to ~per_step seconds
    for _ in range(args.warmup):
        oracle_sample(w, head, per_step)
    vals, rows_total, el_total = [], 0, 0.0
    threads = oracle.num_threads()
    for s in range(args.steps):
        v, rows, el, threads = oracle_sample(w, head, per_step, seed=s + 1)
        vals.append(v)
        rows_total += rows
        el_total += el
    value = 12.0 * rows_total * w.Lk * w.d / el_total / 1e12
    sample = (f"{rows_total} query rows of head 0 over {args.steps} steps (each all {w.Lk} keys), "
              f"{el_total:.1f} s of fp64 oracle time")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el_total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, world):
    in_bytes = w.B * w.H * (2 * w.Lq + 4 * w.Lk) * w.d * w.elem_size
    return {"workload": w.name, "B": w.B, "H": w.H, "Lq": w.Lq, "Lk": w.Lk, "d": w.d, "scale": w.scale,
            "io": w.dtype, "parallelism": "single GPU" if world == 1 else f"{world} independent replicas",
            "l2": (f"inputs larger than L2 ({in_bytes / 1e6:.0f} MB vs {L2_BYTES / 1e6:.0f} MB), no flush"
                   if in_bytes > L2_BYTES else "L2 flushed between steps")}


def run_ours(args, w):
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, local)
    import attention_forward_mode_b200 as ajvp
    ajvp.load_library()

    inp = make_inputs(w, seed=rank, device=dev)
    # entry point: attn_jvp_fwd (bf16 outputs), attn_jvp_fwd_f32out (fp32 outputs) or
    # attn_jvp_fwd_causal (causal mask: FLOPs counted over the visible pairs only)
    # or attn_jvp_fwd_varlen (the heads' tokens packed as 8 sequences of seeded lengths)
    entry_name = {"bf16": "attn_jvp_fwd", "f32out": "attn_jvp_fwd_f32out", "causal": "attn_jvp_fwd_causal",
                  "varlen": "attn_jvp_fwd_varlen"}[args.entry]
    flops = causal_flops(w) if args.entry == "causal" else w.flops
    seq_lens = None
    if args.entry == "varlen":
        import numpy as np
        seq_lens = varlen_lengths(w)
        cu = torch.tensor(np.concatenate([[0], np.cumsum(seq_lens)]), dtype=torch.int32, device=dev)
        flops = 12.0 * w.d * w.B * w.H * float(sum(n * n for n in seq_lens))

        def fwd(q, k, v, tq, tk, tv, scale, o, to, lse, stream):
            ajvp.attn_jvp_fwd_varlen(q[0], k[0], v[0], tq[0], tk[0], tv[0], cu, cu, max(seq_lens), scale,
                                     o=o[0], to=to[0], lse=lse[0], stream=stream)
    else:
        fwd = {"bf16": ajvp.attn_jvp_fwd, "f32out": ajvp.attn_jvp_fwd_f32out,
               "causal": ajvp.attn_jvp_fwd_causal}[args.entry]
    out_dtype = torch.float32 if args.entry == "f32out" else torch.bfloat16
    o = torch.empty(inp["q"].shape, device=dev, dtype=out_dtype)
    to = torch.empty(inp["q"].shape, device=dev, dtype=out_dtype)
    lse = torch.empty((w.B, w.H, w.Lq), device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream(dev)
    in_bytes = sum(t.numel() * t.element_size() for t in inp.values())
    flush = None
    if in_bytes <= L2_BYTES:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def step():
        if flush is not None:
            flush.zero_()
        fwd(inp["q"], inp["k"], inp["v"], inp["tq"], inp["tk"], inp["tv"], w.scale,
                          o=o, to=to, lse=lse, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if ajvp.check_device_status(stream) != ajvp.AJVP_OK:
        raise RuntimeError("kernel wait bound exceeded during warm-up")

    # ---- device-timed region: K launches, events on the launching stream
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    ms_max = max_over_ranks(ms, world, dev)
    status = ajvp.check_device_status(stream)
    if status != ajvp.AJVP_OK:
        raise RuntimeError(f"kernel reported {ajvp.strerror(status)}")
    value = aggregate_value(flops, args.steps, world, ms_max / 1e3)
    per_launch_s = ms / 1e3 / args.steps
    achieved = flops / per_launch_s / 1e12
    # the library's scheduling choice for this call (persistent CTAs for short key sequences)
    n_units = w.B * w.H * ((w.Lq + 127) // 128)
    persistent = (args.entry == "bf16" and (w.Lk + 63) // 64 <= ajvp.DEFAULT_PERSISTENT_KEY_TILES
                  and n_units > torch.cuda.get_device_properties(dev).multi_processor_count)

    # ---- end to end: pinned host inputs -> device -> C ABI -> host, every step
    host_in = {n: t.detach().to("cpu").pin_memory() for n, t in inp.items()}
    host_o = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    host_to = torch.empty(to.shape, dtype=to.dtype).pin_memory()
    host_lse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in (host_o, host_to, host_lse))

    if args.entry == "bf16":
        # the library's host-buffer entry point: head chunks staged through a
        # device workspace, copies in and out overlapped with the kernel
        nh = ajvp.default_heads_per_chunk(w.B * w.H, w.Lq, w.Lk, w.d)
        ws = torch.empty(ajvp.host_workspace_bytes(w.Lq, w.Lk, w.d, nh), dtype=torch.uint8, device=dev)
        e2e_path = f"attn_jvp_fwd_host (pipelined, chunks of {nh} head(s))"

        def e2e_step():
            ajvp.attn_jvp_fwd_host(host_in["q"], host_in["k"], host_in["v"], host_in["tq"], host_in["tk"],
                                   host_in["tv"], w.scale, o=host_o, to=host_to, lse=host_lse, workspace=ws,
                                   stream=stream)
    else:
        e2e_path = f"copy in, {entry_name}, copy out (serial on one stream)"

        def e2e_step():
            for n in inp:
                inp[n].copy_(host_in[n], non_blocking=True)
            fwd(inp["q"], inp["k"], inp["v"], inp["tq"], inp["tk"], inp["tv"], w.scale,
                o=o, to=to, lse=lse, stream=stream)
            host_o.copy_(o, non_blocking=True)
            host_to.copy_(to, non_blocking=True)
            host_lse.copy_(lse, non_blocking=True)

    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ev2, ev3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev2.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    ev3.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(ev2.elapsed_time(ev3), world, dev)
    e2e_value = aggregate_value(flops, e2e_steps, world, e2e_ms / 1e3)

    line = None
    if rank == 0:
        burst, sustained, src = measured_peaks()
        clk = clocks.summary()
        line = {"metric": MASKED_METRIC if args.entry in ("causal", "varlen") else METRIC, "value": value,
                "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": dict(workload_config(w, world), entry=entry_name,
                               **({"flops_per_step": "12·d per visible (query, key) pair"}
                                  if args.entry in ("causal", "varlen") else {}),
                               **({"sequence_lengths": seq_lens} if seq_lens else {})),
                "pct_of_bf16_peak": 100.0 * value / world / burst,
                "roofline": {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                             "frac": achieved / burst,
                             "traffic": committed_traffic(FWD_TRAFFIC_FILES[w.name])
                             if args.entry == "bf16" and w.name in FWD_TRAFFIC_FILES else
                             committed_traffic(F32OUT_TRAFFIC_FILES[w.name])
                             if args.entry == "f32out" and w.name in F32OUT_TRAFFIC_FILES else None,
                             "peak_source": f"{src} bf16 dense (burst) from MEASURED_PEAKS.json"
                             if src == "measured" else "fallback 1.59 PFLOP/s",
                             "kernel": "attn_jvp_fwd_kernel" + (" (persistent form)" if persistent else ""),
                             "algorithmic_flops_per_launch": flops,
                             "algorithmic_bytes_per_launch": w.io_bytes
                             + (4 * w.B * w.H * w.Lq * w.d if args.entry == "f32out" else 0)},  # fp32 O, tO
                "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h, "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
                        "path": e2e_path},
                "gpu_launches": args.steps,
                "clocks": clk}
        # CPU oracle next to the kernel: rank 0 at N = 1 only
        if world == 1 and not args.no_cpu_baseline and args.entry == "causal":
            v, n, el, threads = oracle_sample_causal(w, head0_cpu(inp), args.cpu_seconds)
            line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                    "sample": f"causal sub-problem of the first {n} query rows and keys of head 0 "
                                              f"({el:.1f} s, fp64, OpenMP)"}
        elif world == 1 and not args.no_cpu_baseline and args.entry == "varlen":
            import dataclasses
            b0 = max(range(len(seq_lens)), key=lambda b: seq_lens[b])  # the longest sequence
            a0, n0 = sum(seq_lens[:b0]), seq_lens[b0]
            w0 = dataclasses.replace(w, Lq=n0, Lk=n0)
            v, rows, el, threads = oracle_sample(w0, tuple(x[a0:a0 + n0] for x in head0_cpu(inp)), args.cpu_seconds)
            line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                    "sample": f"{rows} random query rows of sequence {b0} ({n0} tokens) of head 0 "
                                              f"against its keys ({el:.1f} s, fp64, OpenMP)"}
        elif world == 1 and not args.no_cpu_baseline:
            v, rows, el, threads = oracle_sample(w, head0_cpu(inp), args.cpu_seconds)
            line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                    "sample": f"{rows} random query rows of head 0 against all {w.Lk} keys "
                                              f"({el:.1f} s, fp64, OpenMP)"}
        if world == 1 and not args.no_eager and args.entry not in ("causal", "varlen"):
            line["eager_torch_jvp"] = eager_reference(w, inp)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------- backward
def bwd_flops(w) -> float:
    """Backward contraction FLOPs of one (batch, head) set: 15 products of
    2 Lq Lk d each (S, two score-tangent terms, dtO V^T, dO V^T, dtO tV^T,
    two each for dV, dK, dQ and one each for dtV, dtK, dtQ)."""
    return 30.0 * w.B * w.H * w.Lq * w.Lk * w.d


def oracle_bwd_sample(w, full_cpu_head, seconds: float, seed: int = 0):
    """Time the fp64 backward oracle on a prefix sub-problem of one head: the
    first n query rows with every key (a complete backward of an n-row
    problem, 30 n Lk d FLOPs), n sized to about ``seconds``."""
    import oracle
    x = full_cpu_head
    probe = max(4, 2 * oracle.num_threads())

    def run(n):
        t0 = time.perf_counter()
        oracle.attn_jvp_bwd(x["q"][None, :n], x["k"][None], x["v"][None], x["tq"][None, :n], x["tk"][None],
                            x["tv"][None], x["dout"][None, :n], x["dtout"][None, :n], w.scale)
        return time.perf_counter() - t0

    per_row = max(run(probe) / probe, 1e-6)
    n = int(max(1, min(x["q"].shape[0], seconds / per_row)))
    el = run(n)
    return 30.0 * n * w.Lk * w.d / el / 1e12, n, el, oracle.num_threads()


def varlen_lengths(w):
    """The 8 packed sequences of ``--entry varlen`` / ``bwd_varlen``: the
    workload's tokens cut at 7 seeded positions."""
    import numpy as np
    cuts = np.sort(np.random.default_rng(0).choice(np.arange(1, w.Lq), size=7, replace=False))
    return np.diff(np.concatenate([[0], cuts, [w.Lq]])).astype(int).tolist()


def bwd_causal_flops(w) -> float:
    """30 d FLOPs per visible (query, key) pair of the causal mask, summed
    over the heads (the backward's count of ``bwd_flops`` over visible pairs)."""
    return causal_flops(w) * 30.0 / 12.0


def oracle_bwd_sample_causal(w, full_cpu_head, seconds: float):
    """Time the fp64 masked backward oracle on the causal sub-problem made of
    the first n query rows and the first n + Lk - Lq keys of one head (a
    complete n-row causal backward), n sized to about ``seconds``; FLOPs
    30 d per visible pair of that sub-problem."""
    import oracle
    x = full_cpu_head
    off = w.Lk - w.Lq

    def run(n):
        nk = max(1, min(w.Lk, n + off))
        t0 = time.perf_counter()
        oracle.attn_jvp_bwd_causal(x["q"][None, :n], x["k"][None, :nk], x["v"][None, :nk], x["tq"][None, :n],
                                   x["tk"][None, :nk], x["tv"][None, :nk], x["dout"][None, :n],
                                   x["dtout"][None, :n], w.scale)
        return time.perf_counter() - t0, nk

    n = 64
    el, nk = run(n)
    while el < seconds / 4 and n < w.Lq:  # the cost grows like n^2: double until a quarter of the budget
        n = min(w.Lq, 2 * n)
        el, nk = run(n)
    i = torch.arange(n, dtype=torch.float64)
    vis = torch.clamp(i + (nk - n) + 1, 0, nk).sum().item()
    return 30.0 * w.d * vis / el / 1e12, n, el, oracle.num_threads()


def bwd_head0_cpu(inp, cot):
    return {n: t[0, 0].detach().cpu() for n, t in {**inp, **cot}.items()}


def run_reference_bwd(args, w):
    rank, world, local = dist_env()
    if rank != 0:
        return 0
    import oracle
    from attention_forward_mode_b200.workloads import make_cotangents
    oracle.build()
    w0 = w  # the workload named in the line (a packed call's sample is one of its sequences)
    causal = args.entry == "bwd_causal"
    head = bwd_head0_cpu(make_inputs(w, seed=0, device="cpu"), make_cotangents(w, device="cpu"))
    per_step = max(0.5, args.reference_seconds / max(1, args.steps + args.warmup))
    sample_fn = oracle_bwd_sample_causal if causal else oracle_bwd_sample
    if args.entry == "bwd_varlen":
        # packed sequences are independent problems: the longest one stands for the pack
        import dataclasses
        lens = varlen_lengths(w)
        b0 = max(range(len(lens)), key=lambda b: lens[b])
        a0, n0 = sum(lens[:b0]), lens[b0]
        head = {n: t[a0:a0 + n0] for n, t in head.items()}
        w = dataclasses.replace(w, Lq=n0, Lk=n0)
    for _ in range(args.warmup):
        sample_fn(w, head, per_step)
    flops_total, el_total, rows_total, threads = 0.0, 0.0, 0, oracle.num_threads()
    for _ in range(args.steps):
        v, n, el, threads = sample_fn(w, head, per_step)
        flops_total += v * 1e12 * el
        rows_total += n
        el_total += el
    value = flops_total / el_total / 1e12
    what = (f"causal backward sub-problems of the first query rows and keys of head 0" if causal else
            f"backward of the first query rows of head 0 with all {w.Lk} keys"
            + (" of its longest packed sequence" if args.entry == "bwd_varlen" else ""))
    sample = f"{what}, {rows_total} rows over {args.steps} steps, {el_total:.1f} s of fp64 oracle time"
    masked = args.entry in ("bwd_causal", "bwd_varlen")
    line = {"impl": "reference", "metric": BWD_MASKED_METRIC if masked else BWD_METRIC, "value": value,
            "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el_total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(workload_config(w0, world),
                           entry={"bwd": "attn_jvp_bwd", "bwd_causal": "attn_jvp_bwd_causal",
                                  "bwd_varlen": "attn_jvp_bwd_varlen"}[args.entry]),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours_bwd(args, w):
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, local)
    import attention_forward_mode_b200 as ajvp
    from attention_forward_mode_b200.workloads import make_cotangents
    ajvp.load_library()
    names = ("q", "k", "v", "tq", "tk", "tv")
    causal = args.entry == "bwd_causal"
    varlen = args.entry == "bwd_varlen"
    inp = make_inputs(w, seed=rank, device=dev)
    cot = make_cotangents(w, seed=1000 + rank, device=dev)
    stream = torch.cuda.current_stream(dev)
    if varlen:
        # the (batch, head) slabs' tokens packed as 8 sequences, [H, total, d] views
        import numpy as np
        seq_lens = varlen_lengths(w)
        cu = torch.tensor(np.concatenate([[0], np.cumsum(seq_lens)]), dtype=torch.int32, device=dev)
        pk = {n: t.reshape(-1, t.shape[-2], t.shape[-1]) for n, t in {**inp, **cot}.items()}
        o, to, lse, mu = ajvp.attn_jvp_fwd_varlen_stats(*(pk[n] for n in names), cu, cu, max(seq_lens), w.scale,
                                                        stream=stream)
    else:
        fwd = ajvp.attn_jvp_fwd_causal_stats if causal else ajvp.attn_jvp_fwd_stats
        o, to, lse, mu = fwd(*(inp[n] for n in names), w.scale, stream=stream)
    grads = {n: torch.empty_like(inp["q"] if n in ("dq", "dtq") else inp["k"]) for n in ajvp.GRAD_NAMES}
    gpk = {n: g.reshape(-1, g.shape[-2], g.shape[-1]) for n, g in grads.items()}
    ws = torch.empty(ajvp.bwd_workspace_bytes(w.B, w.H, w.Lq, w.Lk), dtype=torch.uint8, device=dev)
    in_bytes = sum(t.numel() * t.element_size() for t in list(inp.values()) + list(cot.values()) + [o, to])
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if in_bytes <= L2_BYTES else None

    def step(which=None):
        if flush is not None:
            flush.zero_()
        if causal:
            ajvp.attn_jvp_bwd_causal(*(inp[n] for n in names), o, to, lse, mu, cot["dout"], cot["dtout"], w.scale,
                                     grads=grads, workspace=ws, stream=stream)
        elif varlen:
            ajvp.attn_jvp_bwd_varlen(*(pk[n] for n in names), o, to, lse, mu, pk["dout"], pk["dtout"], cu, cu,
                                     max(seq_lens), max(seq_lens), w.scale, grads=gpk, workspace=ws, stream=stream)
        else:
            ajvp.attn_jvp_bwd(*(inp[n] for n in names), o, to, lse, mu, cot["dout"], cot["dtout"], w.scale,
                              grads=grads, workspace=ws, stream=stream, step=which)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if ajvp.check_device_status(stream) != ajvp.AJVP_OK:
        raise RuntimeError("kernel wait bound exceeded during warm-up")

    dist = __import__("torch.distributed", fromlist=["barrier"])
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    ms_max = max_over_ranks(ms, world, dev)
    if ajvp.check_device_status(stream) != ajvp.AJVP_OK:
        raise RuntimeError("kernel wait bound exceeded")
    if varlen:
        flops = 30.0 * w.d * w.B * w.H * float(sum(n * n for n in seq_lens))
    else:
        flops = bwd_causal_flops(w) if causal else bwd_flops(w)
    value = aggregate_value(flops, args.steps, world, ms_max / 1e3)
    if causal or varlen:
        return finish_bwd_masked(args, w, rank, world, value, flops, ms_max, clocks, inp, cot,
                                 seq_lens if varlen else None)

    # each of the four kernels alone, K launches each, events on the stream (a split
    # key-side step is its kernel plus the reduction of its partial sums)
    parts = ajvp.bwd_key_split_parts(w.B, w.H, w.Lq, w.Lk)
    per_kernel = []
    nk = max(3, args.steps // 2)
    for i, (kname, fl) in enumerate(BWD_STEPS):
        if parts > 1 and i >= 2:
            kname = f"{kname}, split into {parts} parts + bwd_split_reduce_kernel"
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        step(i)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(nk):
            step(i)
        b.record(stream)
        torch.cuda.synchronize(dev)
        kms = a.elapsed_time(b) / nk
        kfl = fl * w.B * w.H * w.Lq * w.Lk * w.d
        per_kernel.append({"kernel": kname, "ms": kms, "flops": kfl,
                           "tflops": kfl / (kms / 1e3) / 1e12 if fl else None})
    dom = max(per_kernel, key=lambda r: r["ms"])

    # end to end: pinned host inputs -> attn_jvp_bwd_host (head chunks staged through a
    # device workspace, copies overlapped with the kernels) -> host gradients, every step
    dev_in = {**{n: inp[n] for n in names}, "o": o, "to": to, "lse": lse, "mu": mu, **cot}
    host_in = {n: t.detach().to("cpu").pin_memory() for n, t in dev_in.items()}
    host_g = {n: torch.empty(g.shape, dtype=g.dtype).pin_memory() for n, g in grads.items()}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_g.values())
    nh = ajvp.default_bwd_heads_per_chunk(w.B * w.H, w.Lq, w.Lk, w.d)
    host_ws = torch.empty(ajvp.bwd_host_workspace_bytes(w.Lq, w.Lk, w.d, nh), dtype=torch.uint8, device=dev)

    def e2e_step():
        ajvp.attn_jvp_bwd_host(*(host_in[n] for n in names), host_in["o"], host_in["to"], host_in["lse"],
                               host_in["mu"], host_in["dout"], host_in["dtout"], w.scale, grads=host_g,
                               workspace=host_ws, stream=stream)

    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ev2, ev3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev2.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    ev3.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(ev2.elapsed_time(ev3), world, dev)
    e2e_value = aggregate_value(flops, e2e_steps, world, e2e_ms / 1e3)

    line = None
    if rank == 0:
        burst, _, src = measured_peaks()
        achieved = dom["flops"] / (dom["ms"] / 1e3) / 1e12
        line = {"metric": BWD_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": dict(workload_config(w, world), entry="attn_jvp_bwd",
                               flops_per_step="30·Lq·Lk·d per head (minimal contraction count)",
                               key_side_parts=parts),
                "pct_of_bf16_peak": 100.0 * value / world / burst,
                "roofline": {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                             "frac": achieved / burst,
                             "traffic": committed_traffic(BWD_TRAFFIC_FILE, BWD_KERNEL_SOURCES)
                             if w.name == BWD_TRAFFIC_WORKLOAD and dom["kernel"] == BWD_STEPS[2][0] else None,
                             "peak_source": f"{src} bf16 dense (burst) from MEASURED_PEAKS.json"
                             if src == "measured" else "fallback 1.59 PFLOP/s",
                             "kernel": dom["kernel"], "algorithmic_flops_per_launch": dom["flops"],
                             "launch_ms": dom["ms"]},
                "kernels": per_kernel,
                "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                        "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
                        "path": f"attn_jvp_bwd_host (pipelined, chunks of {nh} head(s))"},
                "gpu_launches": (len(BWD_STEPS) + (2 if parts > 1 else 0)) * args.steps,
                "clocks": clocks.summary()}
        if world == 1 and not args.no_cpu_baseline:
            v, n, el, threads = oracle_bwd_sample(w, bwd_head0_cpu(inp, cot), args.cpu_seconds)
            line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                    "sample": f"backward of the first {n} query rows of head 0 with all {w.Lk} keys "
                                              f"({el:.1f} s, fp64, OpenMP)"}
        print(json.dumps(line), flush=True)
    return 0


def finish_bwd_masked(args, w, rank, world, value, flops, ms_max, clocks, inp, cot, seq_lens=None):
    """JSON line of ``--entry bwd_causal`` / ``bwd_varlen``: the masked
    backward timed as one step (four kernels; there is no per-kernel or
    host-buffer entry for it), FLOPs counted over the visible pairs."""
    entry = "attn_jvp_bwd_varlen" if seq_lens else "attn_jvp_bwd_causal"
    if rank == 0:
        burst, _, src = measured_peaks()
        achieved = flops / (ms_max / args.steps / 1e3) / 1e12
        line = {"metric": BWD_MASKED_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic",
                "config": dict(workload_config(w, world), entry=entry,
                               flops_per_step="30·d per visible (query, key) pair",
                               **({"sequence_lengths": seq_lens} if seq_lens else {})),
                "pct_of_bf16_peak": 100.0 * value / world / burst,
                "roofline": {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                             "frac": achieved / burst, "traffic": None,
                             "peak_source": f"{src} bf16 dense (burst) from MEASURED_PEAKS.json"
                             if src == "measured" else "fallback 1.59 PFLOP/s",
                             "kernel": f"{entry} (row statistics and three gradient kernels, one step)",
                             "algorithmic_flops_per_launch": flops},
                "e2e": None,
                "gpu_launches": 4 * args.steps, "clocks": clocks.summary()}
        if world == 1 and not args.no_cpu_baseline and seq_lens:
            import dataclasses
            b0 = max(range(len(seq_lens)), key=lambda b: seq_lens[b])  # the longest sequence
            a0, n0 = sum(seq_lens[:b0]), seq_lens[b0]
            head = {n: t[a0:a0 + n0] for n, t in bwd_head0_cpu(inp, cot).items()}
            v, n, el, threads = oracle_bwd_sample(dataclasses.replace(w, Lq=n0, Lk=n0), head, args.cpu_seconds)
            line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                    "sample": f"backward of the first {n} query rows of sequence {b0} ({n0} tokens) "
                                              f"of head 0 with its keys ({el:.1f} s, fp64, OpenMP)"}
        elif world == 1 and not args.no_cpu_baseline:
            v, n, el, threads = oracle_bwd_sample_causal(w, bwd_head0_cpu(inp, cot), args.cpu_seconds)
            line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                    "sample": f"causal backward of the first {n} query rows and keys of head 0 "
                                              f"({el:.1f} s, fp64, OpenMP)"}
        print(json.dumps(line), flush=True)
    return 0


def eager_reference(w, inp, chunk: int = 8192):
    """torch.func.jvp of softmax(s q k^T) v in the I/O dtype on the GPU,
    looped over heads and 8192-row query chunks (what fits in memory);
    one untimed pass, then one timed pass."""
    def attn(q, k, v):
        return torch.softmax((q @ k.transpose(-1, -2)) * w.scale, dim=-1) @ v

    def one_pass():
        for b in range(w.B):
            for h in range(w.H):
                k, v, tk, tv = (inp[n][b, h] for n in ("k", "v", "tk", "tv"))
                for r0 in range(0, w.Lq, chunk):
                    q = inp["q"][b, h, r0:r0 + chunk]
                    tq = inp["tq"][b, h, r0:r0 + chunk]
                    torch.func.jvp(attn, (q, k, v), (tq, tk, tv))
    try:
        one_pass()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        one_pass()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        return {"value": w.flops / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
                "how": f"torch.func.jvp, {w.dtype}, per head, {chunk}-row query chunks, summed"}
    except Exception as exc:  # e.g. out of memory on a shared GPU
        torch.cuda.empty_cache()
        return {"value": None, "unit": "TFLOP/s", "error": f"{type(exc).__name__}: {exc}"[:200]}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=BENCH_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--reference-seconds", type=float, default=90.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-eager", action="store_true")
    ap.add_argument("--entry", choices=["bf16", "f32out", "causal", "varlen", "bwd", "bwd_causal", "bwd_varlen"],
                    default="bf16",
                    help="f32out: time attn_jvp_fwd_f32out (fp32 outputs, split-bf16 probabilities); "
                         "causal: attn_jvp_fwd_causal; varlen: attn_jvp_fwd_varlen on 8 packed sequences; "
                         "bwd: time the backward pass attn_jvp_bwd; bwd_causal: attn_jvp_bwd_causal; "
                         "bwd_varlen: attn_jvp_bwd_varlen on the 8 packed sequences of varlen")
    ap.add_argument("--heads", type=int, default=None,
                    help="override H (small profiling captures); the JSON config shows the H used")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # timing rule: at least 3 untimed warm-up steps
    w = WORKLOADS[args.workload]
    if args.heads is not None:
        import dataclasses
        w = dataclasses.replace(w, H=args.heads, name=f"{w.name}_h{args.heads}")
    if w.dtype != "bf16" and args.impl == "ours":
        ap.error("the benchmark times the bf16 tensor-core path")
    if args.entry in ("bwd", "bwd_causal", "bwd_varlen"):
        return run_reference_bwd(args, w) if args.impl == "reference" else run_ours_bwd(args, w)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
