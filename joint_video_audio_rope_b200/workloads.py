"""Seeded synthetic workloads: sequence layouts and input tensors.

This module is the only code shared by the CUDA library's callers (tests,
bench) and the fp64 oracle.  It holds configuration and random-number
generation only -- none of the attention, RoPE, pooling or selection
arithmetic.  Inputs are drawn in float32 from numpy's PCG64 with a fixed seed
and, for bf16 workloads, rounded to bfloat16 (round to nearest even) once;
the same bits go to the GPU and to the oracle.  Tensors are drawn in chunks
of tokens, each chunk from its own stream spawned from the workload seed, so
that several threads can draw them and the values still depend on the seed
alone.

Layouts follow the sequence order [conditioning frames (t<0) | video | audio
| text] of one batch item.  Audio tokens use the 21/218 temporal scale that
makes 218 audio tokens span 21 latent frames (SkyReels-V4 digest, novelty 5).
"""
from __future__ import annotations

import os
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import numpy as np

SEG_VIDEO, SEG_AUDIO, SEG_TEXT = 0, 1, 2
ORDER_RASTER, ORDER_BLOCK444 = 0, 1
AUDIO_T_NUM, AUDIO_T_DEN = 21, 218


def video(T, H, W, t0=0, order=ORDER_RASTER):
    return dict(kind=SEG_VIDEO, n_tokens=T * H * W, T=T, H=H, W=W, t0=t0,
                t_num=1, t_den=1, order=order)


def audio(n, t0=0):
    return dict(kind=SEG_AUDIO, n_tokens=n, T=n, H=1, W=1, t0=t0,
                t_num=AUDIO_T_NUM, t_den=AUDIO_T_DEN, order=ORDER_RASTER)


def text(n):
    return dict(kind=SEG_TEXT, n_tokens=n, T=n, H=1, W=1, t0=0, t_num=1,
                t_den=1, order=ORDER_RASTER)


@dataclass
class Workload:
    name: str
    segments: List[dict]
    batch: int
    heads: int
    head_dim: int
    dtype: str                   # "bf16" or "f32"
    seed: int
    qk_std: float                # std of the N(0, std^2) background of Q and K
    v_std: float
    planted_regions: int = 0     # Gaussian "hot" regions added to Q and K
    planted_amp: float = 0.0
    mask: bool = False           # carry a channel-concat mask (never applied)
    sparse: bool = False         # block-sparse video self-attention
    top_k: int = 32
    top_p: float = 0.9
    theta: float = 10000.0
    extra: Dict = field(default_factory=dict)
    plant_v: bool = False        # add the planted regions to V as well
    adaptive: bool = False       # content-adaptive blocks (raster video, planned per step)

    @property
    def n_tokens(self) -> int:
        return sum(s["n_tokens"] for s in self.segments)

    @property
    def n_video(self) -> int:
        """Tokens of the video stream (conditioning frames included)."""
        return sum(s["n_tokens"] for s in self.segments if s["kind"] == SEG_VIDEO)

    @property
    def n_audio(self) -> int:
        return sum(s["n_tokens"] for s in self.segments if s["kind"] == SEG_AUDIO)

    def video_range(self) -> Tuple[int, int]:
        return _kind_range(self.segments, SEG_VIDEO)

    def audio_range(self) -> Tuple[int, int]:
        return _kind_range(self.segments, SEG_AUDIO)

    def text_range(self) -> Tuple[int, int]:
        return _kind_range(self.segments, SEG_TEXT)


def _kind_range(segs, kind):
    start = 0
    lo = hi = None
    for s in segs:
        if s["kind"] == kind:
            if lo is None:
                lo = start
            elif hi != start:
                raise ValueError("segments of one kind must be contiguous")
            hi = start + s["n_tokens"]
        start += s["n_tokens"]
    if lo is None:
        return (0, 0)
    return (lo, hi)


INV_SQRT_128 = float(1.0 / np.sqrt(128.0))

# The five workloads of the benchmark.  Sizes follow the 480p / 720p / 1080p
# 21-latent-frame shapes; 218 audio tokens span the 21 frames.
WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": Workload(
        "tiny_f32", [video(1, 4, 4, t0=-1), video(3, 4, 4), audio(32), text(16)],
        batch=1, heads=2, head_dim=64, dtype="f32", seed=0, qk_std=1.0, v_std=1.0),
    "480p": Workload(
        "480p", [video(21, 30, 52), audio(218), text(512)],
        batch=1, heads=24, head_dim=128, dtype="bf16", seed=1,
        qk_std=INV_SQRT_128, v_std=INV_SQRT_128),
    "720p": Workload(
        "720p", [video(21, 45, 80), audio(218), text(512)],
        batch=1, heads=24, head_dim=128, dtype="bf16", seed=2,
        qk_std=INV_SQRT_128, v_std=INV_SQRT_128),
    "720p_cond_b2": Workload(
        "720p_cond_b2", [video(2, 45, 80, t0=-2), video(21, 45, 80), audio(218), text(512)],
        batch=2, heads=24, head_dim=128, dtype="bf16", seed=3,
        qk_std=INV_SQRT_128, v_std=INV_SQRT_128, mask=True),
    "1080p_sparse": Workload(
        "1080p_sparse", [video(21, 68, 120, order=ORDER_BLOCK444), audio(218)],
        batch=1, heads=24, head_dim=128, dtype="bf16", seed=4,
        qk_std=1.0, v_std=1.0, planted_regions=8, planted_amp=2.0, sparse=True),
    # the 1080p layer with Prism's content-adaptive blocks: raster video whose
    # values V carry the planted regions too (the zones' directional variance
    # decides block volumes and shapes)
    "1080p_adaptive": Workload(
        "1080p_adaptive", [video(21, 68, 120), audio(218)],
        batch=1, heads=24, head_dim=128, dtype="bf16", seed=6,
        qk_std=1.0, v_std=1.0, planted_regions=8, planted_amp=2.0, sparse=True,
        plant_v=True, adaptive=True),
    # the adaptive layer on a quarter of the 1080p grid (profiling size)
    "1080p_adaptive_quarter": Workload(
        "1080p_adaptive_quarter", [video(21, 34, 60), audio(218)],
        batch=1, heads=24, head_dim=128, dtype="bf16", seed=7,
        qk_std=1.0, v_std=1.0, planted_regions=8, planted_amp=2.0, sparse=True,
        plant_v=True, adaptive=True),
    # a quarter of the 1080p grid (17 x 30 -> 17 x 15 blocks per frame slab):
    # the same structure at a size an ncu capture can hold (~2 GB on device)
    "1080p_sparse_quarter": Workload(
        "1080p_sparse_quarter", [video(21, 34, 60, order=ORDER_BLOCK444), audio(218)],
        batch=1, heads=24, head_dim=128, dtype="bf16", seed=5,
        qk_std=1.0, v_std=1.0, planted_regions=8, planted_amp=2.0, sparse=True),
}


def reduced(name: str, T: int, H: int, W: int, n_audio: Optional[int] = None,
            n_text: Optional[int] = None, heads: int = 2, seed_offset: int = 100,
            batch: Optional[int] = None) -> Workload:
    """A smaller workload with the structure of ``name``: every video segment
    gets the grid (T', H, W) with T' = T for the target video and the original
    frame count for conditioning frames."""
    w = WORKLOADS[name]
    segs = []
    for s in w.segments:
        if s["kind"] == SEG_VIDEO:
            tt = s["T"] if s["t0"] < 0 else T
            segs.append(video(tt, H, W, t0=s["t0"], order=s["order"]))
        elif s["kind"] == SEG_AUDIO:
            segs.append(audio(n_audio if n_audio is not None else s["n_tokens"]))
        else:
            segs.append(text(n_text if n_text is not None else s["n_tokens"]))
    return Workload(f"{name}_reduced_{T}x{H}x{W}", segs, batch or w.batch, heads,
                    w.head_dim, w.dtype, w.seed + seed_offset, w.qk_std, w.v_std,
                    w.planted_regions, w.planted_amp, w.mask, w.sparse, w.top_k,
                    w.top_p, w.theta, plant_v=w.plant_v, adaptive=w.adaptive)


# ---------------------------------------------------------------------------
# bf16 helpers (storage conversion only)
# ---------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16, nearest even; returns uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((b >> 16) & 1) + np.uint32(0x7FFF)
    return ((b + r) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# generators
# ---------------------------------------------------------------------------

def _block_major_permutation(T: int, H: int, W: int) -> np.ndarray:
    """Raster index of every token of a T x H x W grid, listed in 4x4x4
    block-major storage order (blocks in (tb, hb, wb) raster order, tokens
    inside a block in (t, h, w) raster order over the block's real extent)."""
    idx = np.arange(T * H * W, dtype=np.int64).reshape(T, H, W)
    parts = []
    for t0 in range(0, T, 4):
        for h0 in range(0, H, 4):
            for w0 in range(0, W, 4):
                parts.append(idx[t0:t0 + 4, h0:h0 + 4, w0:w0 + 4].reshape(-1))
    return np.concatenate(parts)


def _planted_bump(seg: dict, n_regions: int, amp: float, rng) -> np.ndarray:
    """max over regions of amp * exp(-|(x - c) / sigma|^2 / 2) on the grid of
    a video segment, in the segment's storage order (float32, [n_tokens]).
    Centres are uniform in the grid; sigma per axis = extent / 8."""
    T, H, W = seg["T"], seg["H"], seg["W"]
    tt, hh, ww = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    bump = np.zeros((T, H, W), np.float32)
    sig = np.array([T, H, W], np.float64) / 8.0
    for _ in range(n_regions):
        c = rng.uniform(0, 1, 3) * np.array([T, H, W])
        d2 = (((tt - c[0]) / sig[0]) ** 2 + ((hh - c[1]) / sig[1]) ** 2
              + ((ww - c[2]) / sig[2]) ** 2)
        bump = np.maximum(bump, (amp * np.exp(-0.5 * d2)).astype(np.float32))
    flat = bump.reshape(-1)
    if seg["order"] == ORDER_BLOCK444:
        flat = flat[_block_major_permutation(T, H, W)]
    return flat


def _mask(w: Workload, rng) -> np.ndarray:
    """uint8 [B, frames, H, W]: axis-aligned boxes with uniform corners added
    until at least 30% of the tokens are covered."""
    vids = [s for s in w.segments if s["kind"] == SEG_VIDEO]
    F = sum(s["T"] for s in vids)
    H, W = vids[0]["H"], vids[0]["W"]
    m = np.zeros((w.batch, F, H, W), np.uint8)
    for b in range(w.batch):
        while m[b].mean() < 0.30:
            lo = [rng.integers(0, n) for n in (F, H, W)]
            hi = [rng.integers(l, n) + 1 for l, n in zip(lo, (F, H, W))]
            m[b, lo[0]:hi[0], lo[1]:hi[1], lo[2]:hi[2]] = 1
    return m


GEN_CHUNK_TOKENS = 2048  # tokens of one independently seeded generation chunk


def _fill_chunk(out, name_idx, w, seed_seq, t0, t1, std, bump):
    """Draw tokens [t0, t1) of one tensor from its own PCG64 stream (child
    `seed_seq` of the workload seed), scale, add the planted bump, round."""
    rng = np.random.Generator(np.random.PCG64(seed_seq))
    x = rng.standard_normal((w.batch, t1 - t0, w.heads, w.head_dim), dtype=np.float32)
    x *= np.float32(std)
    if bump is not None and (name_idx < 2 or w.plant_v):
        x += bump[None, t0:t1, None, None]
    out[:, t0:t1] = f32_to_bf16_bits(x) if w.dtype == "bf16" else x


def generate(w: Workload, threads: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Q, K, V [B, N, heads, d] (+ mask).  bf16 workloads return uint16 bit
    patterns under 'q','k','v'; f32 workloads return float32 arrays.

    Every tensor is drawn in chunks of GEN_CHUNK_TOKENS tokens (all batch
    items, heads and channels of those tokens), each from its own PCG64
    stream spawned from the workload seed (numpy SeedSequence), so the values
    do not depend on how many threads draw them.  The planted regions and the
    mask have streams of their own."""
    root = np.random.SeedSequence(w.seed)
    n = w.n_tokens
    n_chunks = max(1, -(-n // GEN_CHUNK_TOKENS))
    kids = root.spawn(3 * n_chunks + 2)
    bump = None
    if w.planted_regions:
        rng_b = np.random.Generator(np.random.PCG64(kids[3 * n_chunks]))
        bump = np.zeros(n, np.float32)
        start = 0
        for s in w.segments:
            if s["kind"] == SEG_VIDEO:
                bump[start:start + s["n_tokens"]] = _planted_bump(s, w.planted_regions,
                                                                  w.planted_amp, rng_b)
            start += s["n_tokens"]
    shape = (w.batch, n, w.heads, w.head_dim)
    dt = np.uint16 if w.dtype == "bf16" else np.float32
    out = {name: np.empty(shape, dt) for name in ("q", "k", "v")}
    jobs = []
    for ti, (name, std) in enumerate((("q", w.qk_std), ("k", w.qk_std), ("v", w.v_std))):
        for c in range(n_chunks):
            t0, t1 = c * GEN_CHUNK_TOKENS, min(n, (c + 1) * GEN_CHUNK_TOKENS)
            jobs.append((out[name], ti, w, kids[ti * n_chunks + c], t0, t1, std, bump))
    workers = threads or min(32, os.cpu_count() or 1)
    if workers > 1 and len(jobs) > 1:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(lambda j: _fill_chunk(*j), jobs))
    else:
        for j in jobs:
            _fill_chunk(*j)
    if w.mask:
        out["mask"] = _mask(w, np.random.Generator(np.random.PCG64(kids[3 * n_chunks + 1])))
    return out


def as_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """The exact values a generated tensor holds, as float64."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, np.float64)
