"""The bench's FLOP accounting and workload helpers on the CPU: the causal
counts against brute-force enumeration of the visible (query, key) pairs,
the packed sequences' cut, and the reporting helpers for committed traffic."""
import itertools

import bench
from attention_forward_mode_b200.workloads import WORKLOADS, custom


def _visible_pairs(Lq, Lk):
    # key j is visible to query i iff j <= i + (Lk - Lq)
    return sum(1 for i, j in itertools.product(range(Lq), range(Lk)) if j <= i + (Lk - Lq))


def test_causal_flops_count_visible_pairs():
    for Lq, Lk in [(1, 1), (5, 5), (7, 3), (3, 7), (64, 200), (130, 129), (10, 0)]:
        w = custom(2, 3, Lq, Lk, 128)
        pairs = _visible_pairs(Lq, Lk)
        assert bench.causal_flops(w) == 12.0 * 128 * 2 * 3 * pairs, (Lq, Lk)
        assert bench.bwd_causal_flops(w) == 30.0 * 128 * 2 * 3 * pairs, (Lq, Lk)


def test_causal_square_is_about_half():
    w = WORKLOADS["video_selfattn_b1h12_l32760_d128"]
    full = 12.0 * w.d * w.B * w.H * w.Lq * w.Lk
    L = w.Lq
    assert bench.causal_flops(w) == full * (L + 1) / (2 * L)


def test_bwd_flops_is_fifteen_products():
    w = custom(1, 2, 300, 200, 128)
    assert bench.bwd_flops(w) == 15 * 2.0 * 2 * 300 * 200 * 128


def test_varlen_lengths_cut():
    for name in ("video_selfattn_b1h12_l32760_d128", "image_selfattn_b2h12_l4096_d128"):
        w = WORKLOADS[name]
        a, b = bench.varlen_lengths(w), bench.varlen_lengths(w)
        assert a == b                       # seeded
        assert len(a) == 8 and sum(a) == w.Lq and min(a) >= 1


def test_committed_traffic_tracks_kernel_sources(tmp_path):
    # the figure counts only while the kernel sources' code (comments and spacing
    # aside) hashes to the recorded value
    src = tmp_path / "k.cuh"
    src.write_text("kernel v1\n")
    summary = tmp_path / "summary.md"
    sha = bench.kernel_source_sha([str(src)])
    summary.write_text(f"notes\ntraffic_bytes_per_launch: 12345\nkernel_source_sha: {sha}\n")
    assert bench.committed_traffic(str(summary), [str(src)]) == 12345.0
    src.write_text("kernel  v1 // a comment\n/* and a block\n comment */\n")  # comments, spacing only
    assert bench.committed_traffic(str(summary), [str(src)]) == 12345.0
    src.write_text("kernel v2\n")
    assert bench.committed_traffic(str(summary), [str(src)]) is None
