"""Host-side logic of bench.py (CPU): the metric's FLOP count, the clock-sample summary and the
traffic record.

* Selected tile pairs per (b, h) are V * (P + topk) + P * n_t (every video query tile keeps the P
  prefix tiles and its topk video tiles; every prefix query tile attends to all n_t tiles), each pair
  4 * T * T * D FLOP (Q.K^T and P.V over T-token tiles).  The expected pair counts are worked out here
  by hand from the workloads' geometry (prefix segment lengths -> segment-pure tiles, grid -> 4x4x4
  cubes with partial edges), independently of the oracle's tiling that config_dict calls.
* The clock summary takes the median SM clock and the throttle reasons that were ever active.
* The committed DRAM traffic record belongs to the current attention kernel sources (the bench reports
  no traffic otherwise).
"""
import math

import pytest

import synth

bench = pytest.importorskip("bench")


def by_hand(segments, grid, sparsity, tile=64, cube=(4, 4, 4)):
    P = sum(math.ceil(s / tile) for s in segments)
    V = math.prod(math.ceil(g / c) for g, c in zip(grid, cube))
    k = max(1, min(math.ceil((1 - sparsity) * V), V))
    return P, V, k, V * (P + k) + P * (P + V)


@pytest.mark.parametrize("name,pairs", [("tiny", 68), ("small", 1920), ("480p", 10672), ("768p_s0.9", 180112),
                                        ("768p_s0.8", 312592)])
def test_selected_pairs_and_flop(name, pairs):
    w = synth.workload(name)
    P, V, k, hand = by_hand(w.segments, w.grid, w.sparsity)
    assert hand == pairs
    c = bench.config_dict(w)
    assert (c["n_prefix_tiles"], c["n_video_tiles"], c["topk"]) == (P, V, k)
    assert c["selected_tile_pairs"] == pairs * w.batch * w.heads
    assert c["selected_tflop_per_call"] == pytest.approx(pairs * w.batch * w.heads * 4 * 64 * 64 * w.head_dim / 1e12)


def test_bench_workload_is_21_tflop():
    """The 1344x768 workload at sparsity 0.9: 20 prefix tiles, 1,152 video tiles, topk 116, 21.15 TFLOP
    of selected pairs; with 128-token tiles (4x4x8 cubes) the same work: 10 prefix tiles, 576 video
    tiles, topk 58, each pair four times the FLOPs."""
    c = bench.config_dict(synth.workload("768p_s0.9"))
    assert (c["n_prefix_tiles"], c["n_video_tiles"], c["topk"]) == (20, 1152, 116)
    assert c["selected_tflop_per_call"] == pytest.approx(21.152445497344)
    w = synth.workload("768p_t128_s0.9")
    P, V, k, hand = by_hand(w.segments, w.grid, w.sparsity, tile=128, cube=(4, 4, 8))
    c = bench.config_dict(w)
    assert (c["n_prefix_tiles"], c["n_video_tiles"], c["topk"]) == (P, V, k) == (10, 576, 58)
    assert c["selected_tflop_per_call"] == pytest.approx(21.152445497344)


def test_clock_summary():
    s = bench.ClockSampler(0)
    row = "0, {sm}, 1965, 900.0, 0x{mask}, {hw}, Not Active, Not Active, {cap}"
    s.lines = [row.format(sm=1700, mask="0", hw="Not Active", cap="Not Active"),
               row.format(sm=1800, mask="4", hw="Not Active", cap="Active"),
               row.format(sm=1750, mask="8", hw="Active", cap="Not Active"),
               "garbage line"]
    out = s.summary()
    assert out["sm_mhz"] == 1750 and out["sm_max_mhz"] == 1965 and out["samples"] == 3
    assert out["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert bench.ClockSampler(0).summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_traffic_record_matches_the_kernel_sources():
    """bench.py reports roofline.traffic only while the capture's source hash matches; this keeps the
    record and the attention kernels in step (re-capture after any change to them)."""
    t = bench.measured_attn_traffic()
    assert t is not None and 4.0e9 < t < 2.0e10
