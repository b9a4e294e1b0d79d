"""Host logic of bench.py that needs no GPU: the algorithmic work it divides
by (4 N_q N_kv d H B flops per attention) against the per-step figures of the
workloads, and the rule that a recorded ncu traffic figure is reported only
for the kernel source it was captured from."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from joint_video_audio_rope_b200 import workloads as WL  # noqa: E402


def test_attention_flops_per_step():
    # joint self-attention over the whole sequence and both cross directions,
    # in TFLOP: 480p, 720p, 720p with 2 conditioning frames at batch 2
    want = {"480p": (13.78, 0.176), "720p": (71.59, 0.405), "720p_cond_b2": (171.47, 0.887)}
    for name, (joint, cross) in want.items():
        f = bench.dense_step_flops(WL.WORKLOADS[name])
        assert abs(f["joint"] / 1e12 - joint) < 0.005, (name, f["joint"])
        assert abs(f["cross"] / 1e12 - cross) < 0.0005, (name, f["cross"])
    # the 1080p block-sparse workload's cross-attention (171,360 video tokens)
    f = bench.dense_step_flops(WL.WORKLOADS["1080p_sparse"])
    assert abs(f["cross"] / 1e12 - 0.918) < 0.0005


def test_attn_flops_counts_both_products():
    # QK^T and PV: 2 flops per multiply-add, two contractions
    assert bench.attn_flops(3, 5, 7, 2, 1) == 4.0 * 3 * 5 * 7 * 2


def test_traffic_reported_only_for_the_captured_source(monkeypatch):
    h = bench.kernel_source_hash()
    monkeypatch.setitem(bench.NCU_TRAFFIC, "480p", {"src": h, "bytes": 123})
    assert bench.ncu_traffic("480p") == 123
    monkeypatch.setitem(bench.NCU_TRAFFIC, "480p", {"src": "0" * 16, "bytes": 123})
    assert bench.ncu_traffic("480p") is None
    assert bench.ncu_traffic("no such workload") is None


def test_peak_follows_the_length_of_the_timed_region():
    peaks = {"bf16_tflops": 1638.7, "bf16_tflops_sustained": 1372.3}
    assert bench.pick_peak(peaks, 240.0) == (1638.7, "bf16_tflops")       # a burst
    assert bench.pick_peak(peaks, 2970.0) == (1372.3, "bf16_tflops_sustained")
    assert bench.pick_peak({}, 5000.0)[0] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]


def test_selected_pair_flops_with_block_lengths():
    import numpy as np
    w = WL.WORKLOADS["1080p_adaptive"]
    # two heads' worth: block lengths 64, 128, 256; rows select {0}, {0, 2}, {1}
    w2 = WL.Workload("t", w.segments, 1, 2, 128, "bf16", 0, 1.0, 1.0)
    idx = np.array([[[[0, -1, -1], [0, 2, -1], [1, -1, -1]]] * 2])
    cnt = np.array([[[1, 2, 1]] * 2])
    blen = [np.array([64, 128, 256])]
    pairs = 64 * 64 + 128 * (64 + 256) + 256 * 128
    assert bench.selected_pair_flops(w2, idx, cnt, blen) == 4.0 * 128 * 2 * pairs
