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


def fp32_tie_tol(qbar_i: np.ndarray, kbar: np.ndarray, scale: float, pool_len: int) -> np.ndarray:
    """Per key block j, a bound (natural-log units) on the error of computing
    ln P_j = s_j - max - ln Z in fp32 (unit roundoff u = 2^-24): the pooled
    means are fp32 sums of <= pool_len values (relative error <= pool_len u
    per element, entering s_j twice), the score is a d-term fp32 dot product
    (<= d u sum_c |qbar_c kbar_jc| scale), the shift by the row maximum adds
    u |s_j - max|, and exp and the normaliser a few u.  Blocks whose log
    probabilities lie within the sum of their bounds are fp32 ties."""
    u = 2.0 ** -24
    qbar_i = np.asarray(qbar_i, np.float64)
    kbar = np.asarray(kbar, np.float64)
    a = np.abs(kbar * qbar_i[None, :]).sum(axis=1) * scale
    sc = (kbar @ qbar_i) * scale
    return u * ((kbar.shape[1] + 2 * pool_len) * a + np.abs(sc - sc.max()) + 4.0)


def selection_verdict(got: np.ndarray, ref: np.ndarray, P: np.ndarray, top_k: int,
                      top_p: float, tol: float = 1e-6, ltol: np.ndarray = None) -> str:
    """Classify a selected block set against the oracle's (Prism guide, Method
    section 3: S_i = Top-k(P_i, k) U Top-p(P_i, p)).

    Returns "exact" when the sets are equal, "tie" when they differ only in
    the way fp32 rounding can legitimately move the cutoff, and "mismatch"
    otherwise.  With the oracle's ranking (P descending, lower id first) and
    n_k = min(k, n) and n_p the shortest prefix whose cumulative sum reaches
    p, the selected size is m = max(n_k, n_p).  Two effects of fp32 are
    allowed, and nothing else:

    * the top-p crossing moves by one block when the cumulative sum that
      decides it is within the mass tolerance of p (n_p - 1 if the sum before
      the crossing block is, n_p + 1 if the sum including it is);
    * at the boundary of a set of size m, blocks whose probability is tied
      with the m-th ranked probability may be swapped for one another.

    Ties: with ``ltol`` (per-block bounds on the fp32 error of ln P_j, see
    ``fp32_tie_tol``) block j is tied with the cutoff block c when
    |ln P_j - ln P_c| <= ltol_j + ltol_c, and the mass tolerance is
    sum_j P_j ltol_j + tol; without it, |P_j - P_c| <= tol P_c and tol.
    So for some allowed size m the GPU set must hold exactly m blocks, every
    block ranked clearly above the m-th, and no block clearly below it: the
    top-k blocks and every block above the cutoff must match exactly.
    """
    g = set(np.asarray(got).tolist())
    r = set(np.asarray(ref).tolist())
    if g == r:
        return "exact"
    P = np.asarray(P, np.float64)
    n = len(P)
    if len(g) != len(np.asarray(got)) or any(j < 0 or j >= n for j in g):
        return "mismatch"  # duplicates or ids out of range
    order = sorted(range(n), key=lambda j: (-P[j], j))
    csum = np.cumsum(P[order])
    if ltol is not None:
        ltol = np.asarray(ltol, np.float64)
        mtol = float((P * ltol).sum()) + tol
    else:
        mtol = tol
    n_k = min(max(top_k, 0), n)
    hit = np.nonzero(csum >= top_p)[0]
    n_p = int(hit[0]) + 1 if len(hit) else n
    sizes = {max(n_k, n_p)}
    if n_p >= 2 and abs(csum[n_p - 2] - top_p) <= mtol:
        sizes.add(max(n_k, n_p - 1))
    if n_p < n and abs(csum[n_p - 1] - top_p) <= mtol:
        sizes.add(max(n_k, n_p + 1))
    with np.errstate(divide="ignore"):
        lp = np.log(P)
    for m in sizes:
        if len(g) != m or m == 0:
            continue
        c = order[m - 1]
        if ltol is not None:
            band = ltol + ltol[c]
            above = {j for j in range(n) if lp[j] > lp[c] + band[j]}
            below = {j for j in range(n) if lp[j] < lp[c] - band[j]}
        else:
            pm = P[c]
            above = {j for j in range(n) if P[j] > pm * (1 + tol)}
            below = {j for j in range(n) if P[j] < pm * (1 - tol)}
        if above <= g and not (g & below):
            return "tie"
    return "mismatch"


def selection_matches(got, ref, P, top_k: int, top_p: float, tol: float = 1e-6,
                      ltol: np.ndarray = None) -> bool:
    """True unless ``selection_verdict`` says "mismatch"."""
    return selection_verdict(got, ref, P, top_k, top_p, tol, ltol) != "mismatch"
