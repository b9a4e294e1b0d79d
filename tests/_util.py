"""Shared test helpers: oracle layouts from workload segments, host<->device
transfer of generated inputs, and the comparison metrics of the parity bar
(max-abs and relative-L2 error)."""
from __future__ import annotations

import math

import numpy as np

import oracle as O
from joint_video_audio_rope_b200 import workloads as WL

BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
F32_TOL = 1e-5


def oracle_layout(segments) -> "O.Layout":
    return O.Layout([O.Segment(s["kind"], s["n_tokens"], s["T"], s["H"], s["W"], s["t0"],
                               s["t_num"], s["t_den"], s["order"]) for s in segments])


def rope_bands(head_dim):
    dh = 2 * (head_dim // 6)
    return head_dim - 2 * dh, dh, dh


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Values rounded to bfloat16 (via float32, nearest even), as float64.

    Models the bf16 storage of an intermediate tensor between two steps of
    the path (e.g. the RoPE output that the attention step reads); the
    rounding is done by the test on the oracle's own values."""
    return WL.bf16_bits_to_f32(WL.f32_to_bf16_bits(np.asarray(x, np.float32))).astype(np.float64)


def to_device(x: np.ndarray, dtype: str):
    import torch
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def to_host_f64(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy().astype(np.float64)


def errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    max_abs = float(np.max(np.abs(got - ref))) if got.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got - ref))
    return max_abs, rel


def assert_close(got, ref, dtype: str, what: str = ""):
    max_abs, rel = errors(got, ref)
    if dtype == "bf16":
        assert max_abs <= BF16_MAX_ABS and rel <= BF16_REL_L2, \
            f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    else:
        assert max_abs <= F32_TOL, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def selection_matches(got: np.ndarray, ref: np.ndarray, P: np.ndarray, top_k: int, top_p: float,
                      tol: float = 1e-6) -> bool:
    """True if the GPU set equals the oracle set, or differs only in blocks
    tied with the cutoff within fp32 resolution: a differing block j is
    excused when |P_j - P_cut| <= tol * P_cut, where P_cut is the smallest
    probability the oracle selected; the whole row is excused when the
    oracle's cumulative sum at its top-p cutoff is within tol of p."""
    g, r = set(got.tolist()), set(ref.tolist())
    if g == r:
        return True
    order = sorted(range(len(P)), key=lambda j: (-P[j], j))
    n_sel = len(r)
    p_cut = P[order[n_sel - 1]]
    csum = np.cumsum(P[order])
    n_k = min(top_k, len(P))
    if n_sel > n_k:  # top-p decided the size
        if abs(csum[n_sel - 1] - top_p) <= tol or (n_sel >= 2 and abs(csum[n_sel - 2] - top_p) <= tol):
            return True
    for j in g ^ r:
        if abs(P[j] - p_cut) > tol * p_cut:
            return False
    return True
