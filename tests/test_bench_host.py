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
