"""Plain fp64 CPU oracle for the joint video/audio attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it.  It shares no code, table or helper with the CUDA
library; the only thing both sides share is the seeded input generator, which
holds none of the method's arithmetic.

Every function is written straight from the definitions, in float64, with no
blocking, fusion or reordering beyond what the definition states, so that a
reader can check it against the sources by eye:

* Sources (cited by page title and section):
  - [SKY-D] "SkyReels-V4: Multi-modal Video-Audio Generation, Inpainting and
    Editing model" -- Chinese digest of arXiv 2602.21818: workflow steps 1-6
    and the list of novelties (4th: time-offset 3D RoPE with negative
    temporal indices; 5th: audio RoPE frequency scaling 21/218).
  - [SKY-B] "SkyReels-V4: dual-stream MMDiT ..." -- trdm.cn blog, sections
    2.1 (dual stream then single stream, joint self-attention), 2.2
    (bidirectional audio<->video cross-attention in every block; 21 video
    frames aligned with 218 audio tokens through RoPE frequency scaling) and
    4.2 (the Refiner refines only the target region of a spatial mask).
  The digest's step 3 also names the reinforced text cross-attention (video
  queries over the text embedding) and its step 4 the flow-matching input,
  target and loss.
  - [PRISM] "Prism: dynamic sparse attention for native 2K joint video-audio
    generation" -- reading guide of arXiv 2610.05416, Method section 3
    (mean-pooled key blocks, block probabilities P_i, and the attended set
    S_i = Top-k(P_i, k) U Top-p(P_i, p)); scope rule in the Method preamble
    (only video self-attention is sparsified, cross-attention stays dense);
    Key ideas and Method sections 1-2 (8x8x8 macro-zones, the dual-guidance
    variation indicator g_d, block volumes B in {64, 128, 256} from a density
    rho against tau_128 = 0.5 and tau_256 = 0.25, and the block shape nearest
    to the optimal log-edges l*_d among 16 candidates).

Readings where the sources are silent are stated at each function; the
complete list is kept with the design notes of the repository.

Pins: every function here is checked by ``tests/test_oracle_*.py`` against
closed forms, invariants, worked values and brute force -- never against the
CUDA path.  The model-level output beyond attention is not computed here.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Sequence, Tuple

import numpy as np

SEG_VIDEO = 0
SEG_AUDIO = 1
SEG_TEXT = 2

ORDER_RASTER = 0
ORDER_BLOCK444 = 1

BLOCK_EDGE = 4  # 4x4x4 token blocks of the sparse mode


@dataclass
class Segment:
    """One contiguous run of tokens of a per-batch sequence.

    kind     : SEG_VIDEO / SEG_AUDIO / SEG_TEXT
    n_tokens : number of tokens in the run
    T, H, W  : video grid (T frames of H x W latent tokens); unused otherwise
    t0       : first temporal index; negative for conditioning/reference
               latents ([SKY-D] step 1: reference latents are concatenated in
               time and told apart from the target by negative time indices)
    t_num, t_den : audio temporal scale t = t0 + j * t_num / t_den
               ([SKY-D] novelty 5: 218 audio tokens span 21 latent frames)
    order    : ORDER_RASTER or ORDER_BLOCK444 (video only)
    """

    kind: int
    n_tokens: int
    T: int = 0
    H: int = 0
    W: int = 0
    t0: int = 0
    t_num: int = 1
    t_den: int = 1
    order: int = ORDER_RASTER


@dataclass
class Layout:
    segments: List[Segment] = field(default_factory=list)

    @property
    def n_tokens(self) -> int:
        return sum(s.n_tokens for s in self.segments)


# ---------------------------------------------------------------------------
# a1: positions
# ---------------------------------------------------------------------------

def _block_major_coords(T: int, H: int, W: int) -> np.ndarray:
    """(t, h, w) of every token of a T x H x W grid stored block-major.

    Blocks of 4x4x4 tokens are visited in (tb, hb, wb) raster order; inside a
    block the tokens are visited in (t, h, w) raster order over the block's
    real extent.  Blocks on the far edge of an axis that does not divide by 4
    are short and hold only their real tokens (no padding in memory).
    """
    e = BLOCK_EDGE
    out = []
    for tb in range(-(-T // e)):
        for hb in range(-(-H // e)):
            for wb in range(-(-W // e)):
                for t in range(tb * e, min(T, tb * e + e)):
                    for h in range(hb * e, min(H, hb * e + e)):
                        for w in range(wb * e, min(W, wb * e + e)):
                            out.append((t, h, w))
    return np.asarray(out, dtype=np.float64).reshape(-1, 3)


def positions(layout: Layout) -> np.ndarray:
    """Per-token RoPE positions (t, h, w) as float64, shape [N, 3].

    * video, raster order: token n -> (t0 + n // (H W), (n // W) % H, n % W)
    * video, block-major: see ``_block_major_coords``; t shifted by t0
    * audio token j -> (t0 + j * t_num / t_den, 0, 0)       [SKY-D] novelty 5
    * text -> (0, 0, 0)   (reading: the sources give text no 3D position)
    """
    rows = []
    for s in layout.segments:
        if s.kind == SEG_VIDEO:
            if s.n_tokens != s.T * s.H * s.W:
                raise ValueError("video segment size != T*H*W")
            if s.order == ORDER_RASTER:
                n = np.arange(s.n_tokens)
                p = np.stack([s.t0 + n // (s.H * s.W), (n // s.W) % s.H, n % s.W], 1)
                p = p.astype(np.float64)
            else:
                p = _block_major_coords(s.T, s.H, s.W)
                p[:, 0] += s.t0
            rows.append(p)
        elif s.kind == SEG_AUDIO:
            j = np.arange(s.n_tokens, dtype=np.float64)
            p = np.zeros((s.n_tokens, 3))
            p[:, 0] = s.t0 + j * s.t_num / s.t_den
            rows.append(p)
        elif s.kind == SEG_TEXT:
            rows.append(np.zeros((s.n_tokens, 3)))
        else:
            raise ValueError("unknown segment kind")
    if not rows:
        return np.zeros((0, 3))
    return np.concatenate(rows, 0)


# ---------------------------------------------------------------------------
# a2: 3D RoPE
# ---------------------------------------------------------------------------

def rope_bands(head_dim: int) -> Tuple[int, int, int]:
    """Channel split (d_t, d_h, d_w) of the 3D RoPE.

    Reading: h and w get 2*floor(d/6) channels each and t the rest, which is
    44/42/42 at d=128 and 24/20/20 at d=64.
    """
    dh = 2 * (head_dim // 6)
    return head_dim - 2 * dh, dh, dh


def rope(x: np.ndarray, pos: np.ndarray, theta: float = 10000.0,
         bands: Tuple[int, int, int] | None = None) -> np.ndarray:
    """Rotate every head of x by its token's (t, h, w) position.

    x   : [..., N, heads, d] (any float dtype; computed in float64)
    pos : [N, 3]
    Channels are split into consecutive bands [t | h | w]; inside band b of
    width d_b, channel pair (2i, 2i+1) -- pairs interleaved, i counted from
    the band start -- is treated as the complex number x_2i + 1j*x_2i+1 and
    multiplied by exp(1j * pos_b * theta**(-2i/d_b)).
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    if bands is None:
        bands = rope_bands(d)
    if sum(bands) != d or any(b % 2 for b in bands):
        raise ValueError("bad RoPE bands")
    z = x[..., 0::2] + 1j * x[..., 1::2]            # [..., N, heads, d/2]
    angle = np.zeros((pos.shape[0], d // 2))
    start = 0
    for axis, db in enumerate(bands):
        i = np.arange(db // 2, dtype=np.float64)
        omega = theta ** (-2.0 * i / db)
        angle[:, start // 2:(start + db) // 2] = pos[:, axis:axis + 1] * omega[None, :]
        start += db
    z = z * np.exp(1j * angle)[:, None, :]
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


# ---------------------------------------------------------------------------
# a3 / a4: attention
# ---------------------------------------------------------------------------

def attn(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """softmax(q k^T * scale) v for one head, float64, no mask.

    q [Nq, d], k [Nk, d], v [Nk, dv] -> (o [Nq, dv], lse [Nq]) where lse is
    the natural-log sum of exp of the scaled scores of each row.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    s = (q @ k.T) * scale
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    o = (e @ v) / l
    lse = (m + np.log(l))[:, 0]
    return o, lse


def attn_bshd(q, k, v, scale):
    """attn for every (batch, head) of [B, N, H, d] tensors."""
    q = np.asarray(q, np.float64)
    B, Nq, H, _ = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, Nq, H, dv))
    lse = np.zeros((B, Nq, H))
    for b in range(B):
        for h in range(H):
            o[b, :, h], lse[b, :, h] = attn(q[b, :, h], k[b, :, h], v[b, :, h], scale)
    return o, lse


def joint_attn(q, k, v, scale):
    """Joint self-attention over the whole concatenated sequence.

    [SKY-D] step 3 and [SKY-B] 2.1: video(/audio) and text tokens are
    projected separately and then attend jointly in one softmax; the
    dual-stream and single-stream blocks run the same attention math.  The
    binary mask M of step 2 is an input channel, not an attention mask, so it
    does not enter here.
    """
    return attn_bshd(q, k, v, scale)


def av_cross_attn(qv, kv, vv, qa, ka, va, scale):
    """Bidirectional audio<->video cross-attention ([SKY-D] step 3,
    [SKY-B] 2.2): video queries attend to the audio keys/values and audio
    queries attend to the video keys/values.  Returns (o_video, o_audio)."""
    o_v, _ = attn_bshd(qv, ka, va, scale)
    o_a, _ = attn_bshd(qa, kv, vv, scale)
    return o_v, o_a


def text_cross_attn(qv, kt, vt, scale):
    """Reinforced text cross-attention ([SKY-D] step 3: in every layer the
    video tokens query the text embedding): softmax(qv kt^T * scale) vt per
    (batch, head), no mask.  Returns o_video."""
    o_v, _ = attn_bshd(qv, kt, vt, scale)
    return o_v


def masked_rows(layout: Layout, mask: np.ndarray) -> List[np.ndarray]:
    """Per batch item, the sequence indices of the video tokens whose mask
    value is non-zero, in sequence order.  ``mask`` is [B, F, H, W] over the
    frames of all video segments in sequence order (the binary mask M of
    [SKY-D] step 2); video segments are in raster order."""
    out = []
    for b in range(mask.shape[0]):
        rows = []
        start, frame = 0, 0
        for s in layout.segments:
            if s.kind == SEG_VIDEO:
                if s.order != ORDER_RASTER:
                    raise ValueError("masked rows need raster-order video segments")
                for t in range(s.T):
                    for h in range(s.H):
                        for w in range(s.W):
                            if mask[b, frame + t, h, w] != 0:
                                rows.append(start + (t * s.H + h) * s.W + w)
                frame += s.T
            start += s.n_tokens
        out.append(np.array(rows, dtype=np.int64))
    return out


def masked_joint_attn(q, k, v, o_init, rows, scale):
    """Mask-guided region-restricted attention ([SKY-B] 4.2: with a spatial
    mask the Refiner refines only the target region): the rows ``rows[b]`` of
    the output get their joint-attention row over every key of batch item b;
    every other row keeps its value from ``o_init``."""
    o = np.array(o_init, dtype=np.float64, copy=True)
    for b in range(q.shape[0]):
        r = rows[b]
        if len(r) == 0:
            continue
        for h in range(q.shape[2]):
            o[b, r, h], _ = attn(q[b, r, h], k[b, :, h], v[b, :, h], scale)
    return o


def flow_noise(z0, eps, t):
    """Flow-matching input and velocity target of one stream ([SKY-D] step 4):
    z_t = t z_0 + (1 - t) eps for each batch item's time t[b], and the
    velocity the model is trained to predict, z_0 - eps.  Arrays are [B, ...];
    returns (z_t, target) in float64."""
    z0 = np.asarray(z0, np.float64)
    eps = np.asarray(eps, np.float64)
    tb = np.asarray(t, np.float64).reshape((-1,) + (1,) * (z0.ndim - 1))
    return tb * z0 + (1.0 - tb) * eps, z0 - eps


def flow_loss(v, z0, eps):
    """The stream's loss term per batch item ([SKY-D] step 4): the squared
    L2 norm || v - (z_0 - eps) ||^2 over the item's values, float64 [B]."""
    d = np.asarray(v, np.float64) - (np.asarray(z0, np.float64) - np.asarray(eps, np.float64))
    return (d.reshape(d.shape[0], -1) ** 2).sum(axis=1)


# ---------------------------------------------------------------------------
# a5 - a7: block-sparse mode
# ---------------------------------------------------------------------------

def video_blocks(T: int, H: int, W: int):
    """Token ranges of the 4x4x4 blocks of a block-major video segment.

    Returns a list of (start, length) in block order (tb, hb, wb raster);
    a block's tokens are contiguous in the block-major storage."""
    e = BLOCK_EDGE
    out = []
    start = 0
    for tb in range(-(-T // e)):
        for hb in range(-(-H // e)):
            for wb in range(-(-W // e)):
                n = ((min(T, tb * e + e) - tb * e) * (min(H, hb * e + e) - hb * e)
                     * (min(W, wb * e + e) - wb * e))
                out.append((start, n))
                start += n
    return out


def pool(x: np.ndarray, blocks) -> np.ndarray:
    """Mean over the real tokens of each block ([PRISM] Method 3: keys are
    mean-pooled into block representatives; the query is pooled the same way
    -- a reading).  x [B, N, H, d] -> [B, H, nblocks, d] float64."""
    x = np.asarray(x, np.float64)
    B, _, Hh, d = x.shape
    out = np.zeros((B, Hh, len(blocks), d))
    for i, (s, n) in enumerate(blocks):
        out[:, :, i, :] = x[:, s:s + n].mean(axis=1)
    return out


def select_from_probs(P: np.ndarray, top_k: int, top_p: float) -> np.ndarray:
    """The attended set S_i = Top-k(P_i, k) U Top-p(P_i, p) of one row of
    block probabilities ([PRISM] Method 3).

    Blocks are ordered by P descending, ties by block id ascending.  Top-k
    takes the first min(k, n) blocks; Top-p takes the shortest prefix whose
    cumulative probability reaches p (the block that crosses p is included;
    if rounding keeps the sum below p, every block).  S_i is their union,
    returned in ascending block id.
    """
    P = np.asarray(P, np.float64)
    n = P.shape[0]
    order = sorted(range(n), key=lambda j: (-P[j], j))
    n_k = min(top_k, n)
    csum = 0.0
    n_p = n
    for r, j in enumerate(order):
        csum += P[j]
        if csum >= top_p:
            n_p = r + 1
            break
    chosen = order[:max(n_k, n_p)]
    return np.asarray(sorted(chosen), dtype=np.int64)


def select_row(qbar_i: np.ndarray, kbar: np.ndarray, top_k: int, top_p: float,
               scale: float) -> np.ndarray:
    """Attended key-block set of one query block ([PRISM] Method 3):
    P_i = softmax_j(qbar_i . kbar_j * scale), then ``select_from_probs``."""
    return select_from_probs(block_probs(qbar_i, kbar, scale), top_k, top_p)


def select_rows(qbar: np.ndarray, kbar: np.ndarray, top_k: int, top_p: float,
                scale: float) -> List[np.ndarray]:
    """``select_row`` for every query block of one (batch, head), for many
    rows at once: qbar [nq, d], kbar [nk, d] -> list of nq int arrays.

    The same definition written with array steps: the block softmax of every
    row, the ranking by a stable sort of -P (equal probabilities keep
    ascending block ids), the running sum along the ranking, the first
    position where it reaches p (every block if none), and the union with the
    first min(k, n) ranked blocks, returned in ascending id.
    """
    s = (np.asarray(qbar, np.float64) @ np.asarray(kbar, np.float64).T) * scale
    e = np.exp(s - s.max(axis=1, keepdims=True))
    P = e / e.sum(axis=1, keepdims=True)
    n = P.shape[1]
    order = np.argsort(-P, axis=1, kind="stable")
    csum = np.cumsum(np.take_along_axis(P, order, axis=1), axis=1)
    reached = csum >= top_p
    n_p = np.where(reached.any(axis=1), reached.argmax(axis=1) + 1, n)
    n_sel = np.maximum(min(top_k, n), n_p)
    return [np.sort(order[i, :n_sel[i]]).astype(np.int64) for i in range(P.shape[0])]


def block_probs(qbar_i, kbar, scale):
    """P_i of ``select_row`` (exposed for tie analysis in the tests)."""
    s = (kbar @ qbar_i) * scale
    e = np.exp(s - s.max())
    return e / e.sum()


def block_select(qbar, kbar, top_k, top_p, scale):
    """``select_row`` for every (batch, head, query block).

    qbar, kbar [B, H, nblk, d] -> nested list sel[b][h][i] of int arrays."""
    B, Hh, nq, _ = qbar.shape
    return [[[select_row(qbar[b, h, i], kbar[b, h], top_k, top_p, scale)
              for i in range(nq)] for h in range(Hh)] for b in range(B)]


def sparse_attn_rows(q, k, v, blocks, sel, scale, b: int, h: int, qblk: int):
    """Sparse attention for the tokens of one query block: the tokens of
    query block ``qblk`` attend only to the tokens of the key blocks in
    ``sel`` (the attended set S_i), with one softmax over all of them
    ([PRISM] Method 3, online-softmax attention over S_i)."""
    s0, n = blocks[qblk]
    kk = np.concatenate([k[b, blocks[j][0]:blocks[j][0] + blocks[j][1], h] for j in sel], 0)
    vv = np.concatenate([v[b, blocks[j][0]:blocks[j][0] + blocks[j][1], h] for j in sel], 0)
    o, lse = attn(q[b, s0:s0 + n, h], kk, vv, scale)
    return o, lse


def sparse_attn(q, k, v, blocks, sel, scale):
    """``sparse_attn_rows`` for every (batch, head, query block);
    q, k, v [B, N, H, d] block-major; sel as returned by block_select."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, N, Hh, _ = q.shape
    o = np.zeros((B, N, Hh, v.shape[-1]))
    for b in range(B):
        for h in range(Hh):
            for i, (s0, n) in enumerate(blocks):
                o[b, s0:s0 + n, h], _ = sparse_attn_rows(q, k, v, blocks, sel[b][h][i],
                                                         scale, b, h, i)
    return o


# ---------------------------------------------------------------------------
# Prism content-adaptive block shapes ([PRISM] Key ideas; Method 1 and 2)
# ---------------------------------------------------------------------------

ZONE = (8, 8, 8)          # Z_T x Z_H x Z_W macro-zone ([PRISM] Key ideas)
TAU_128 = 0.5             # density threshold below which B(m) = 128 ([PRISM] Method 2)
TAU_256 = 0.25            # density threshold below which B(m) = 256
EPS_G = 1e-6              # the epsilon of g_d (reading: a small constant)
VOLUMES = (64, 128, 256)  # B(m)


def shape_candidates(volume: int) -> List[Tuple[int, int, int]]:
    """The candidate block shapes C_B of one volume ([PRISM] Key ideas: 16
    shapes over the volumes {64, 128, 256}).

    Reading: the edges (b_T, b_H, b_W) are powers of two from 2 to the zone
    edge 8 with product B; that gives 7 + 6 + 3 = 16 shapes, the count the
    guide states.  Listed in ascending lexicographic order of the edges, the
    order that breaks distance ties."""
    out = []
    for bt in (2, 4, 8):
        for bh in (2, 4, 8):
            for bw in (2, 4, 8):
                if bt * bh * bw == volume:
                    out.append((bt, bh, bw))
    return out


def macro_zones(T: int, H: int, W: int, zone=ZONE):
    """Macro-zones of a T x H x W token volume ([PRISM] Key ideas), in
    (zt, zh, zw) raster order, as (t0, h0, w0, et, eh, ew).  Reading: zones on
    the far edge of an axis that the zone edge does not divide are short
    (they hold only the real tokens)."""
    out = []
    for t0 in range(0, T, zone[0]):
        for h0 in range(0, H, zone[1]):
            for w0 in range(0, W, zone[2]):
                out.append((t0, h0, w0, min(zone[0], T - t0), min(zone[1], H - h0),
                            min(zone[2], W - w0)))
    return out


def directional_variance(x: np.ndarray) -> np.ndarray:
    """sigma^2_d of one zone for d = T, H, W ([PRISM] Method 1).

    x [Z_T, Z_H, Z_W, D]: the zone's features.  For axis d, the slice means
    xbar^(d)_i average x over the zone's tokens with index i along d (the
    other two axes); mu^(d) is the mean of those slice means over i; and
    sigma^2_d = (1/D) sum_c (1/Z_d) sum_i (xbar^(d)_{i,c} - mu^(d)_c)^2."""
    x = np.asarray(x, np.float64)
    D = x.shape[3]
    out = np.zeros(3)
    for d in range(3):
        other = tuple(a for a in range(3) if a != d)
        xbar = x.mean(axis=other)             # [Z_d, D]
        mu = xbar.mean(axis=0)                # [D]
        out[d] = ((xbar - mu[None, :]) ** 2).mean(axis=0).sum() / D
    return out


def _ratio(sig: np.ndarray) -> np.ndarray:
    """sigma^2_d / sum_d' sigma^2_d'; all zero when the sum is zero (reading)."""
    tot = sig.sum()
    return sig / tot if tot > 0 else np.zeros(3)


def zone_indicators(v: np.ndarray, a: np.ndarray | None, T: int, H: int, W: int,
                    eps: float = EPS_G):
    """The dual-guidance indicator of every macro-zone ([PRISM] Method 1).

    v : [T, H, W, D] value features of one video (D = heads x head_dim)
    a : [T, H, W] or None: the A->V cross-attention output norms
        a_{t,h,w} = ||h_{t,h,w}||_2 cached from the preceding layer; None
        means no audio guidance (abar = 0).
    Per zone m:
      r_{v,d}(m)   = sigma^2_{v,d}(m) / sum_d' sigma^2_{v,d'}(m)
      vhat_{a,d}(m) = sigma^2_{a,d}(m) / sum_d' sigma^2_{a,d'}(m)  (reading:
                      the directional variance of the norms, normalised like r)
      abar(m)      = mean of a over the zone / max over zones of that mean
                      (reading: the coupling strength, normalised to [0, 1])
      g_d(m)       = r_{v,d}(m) + abar(m) * vhat_{a,d}(m) + eps
      rho(m)       = sum_d sigma^2_{v,d}(m) / max over zones of that sum
                      (reading: the normalised spatio-temporal information
                      density of Method 2)
    Returns (zones, g [nz, 3], rho [nz], abar [nz])."""
    zones = macro_zones(T, H, W)
    nz = len(zones)
    sig_v = np.zeros((nz, 3))
    sig_a = np.zeros((nz, 3))
    a_mean = np.zeros(nz)
    for m, (t0, h0, w0, et, eh, ew) in enumerate(zones):
        sig_v[m] = directional_variance(v[t0:t0 + et, h0:h0 + eh, w0:w0 + ew])
        if a is not None:
            az = np.asarray(a, np.float64)[t0:t0 + et, h0:h0 + eh, w0:w0 + ew]
            sig_a[m] = directional_variance(az[..., None])
            a_mean[m] = az.mean()
    amax = a_mean.max() if nz else 0.0
    abar = a_mean / amax if amax > 0 else np.zeros(nz)
    tot = sig_v.sum(axis=1)
    tmax = tot.max() if nz else 0.0
    rho = tot / tmax if tmax > 0 else np.zeros(nz)
    g = np.zeros((nz, 3))
    for m in range(nz):
        g[m] = _ratio(sig_v[m]) + abar[m] * _ratio(sig_a[m]) + eps
    return zones, g, rho, abar


def block_volume(rho: float) -> int:
    """B(m) from the density rho(m) against tau_128 = 0.5 and tau_256 = 0.25
    ([PRISM] Method 2).  Reading: dense zones keep the finest blocks --
    B = 64 for rho >= tau_128, 128 for tau_256 <= rho < tau_128, 256 below."""
    if rho >= TAU_128:
        return 64
    if rho >= TAU_256:
        return 128
    return 256


def optimal_log_edges(g: np.ndarray, volume: int) -> np.ndarray:
    """l*_d = -1/2 log2 g_d + 1/3 (S + 1/2 sum_d' log2 g_d'), S = log2 B(m):
    the minimiser of sum_d g_d (b_d^2 - 1) subject to prod_d b_d = B(m), in
    log2 space (b*_d proportional to g_d^(-1/2)) ([PRISM] Method 2)."""
    lg = np.log2(np.asarray(g, np.float64))
    S = math.log2(volume)
    return -0.5 * lg + (S + 0.5 * lg.sum()) / 3.0


def choose_shape(g: np.ndarray, volume: int) -> Tuple[int, int, int]:
    """The candidate of C_B(m) at the smallest Euclidean distance from l*
    in log2 space ([PRISM] Method 2); ties go to the earlier candidate."""
    ls = optimal_log_edges(g, volume)
    best, best_d = None, None
    for c in shape_candidates(volume):
        d = sum((math.log2(c[i]) - ls[i]) ** 2 for i in range(3))
        if best_d is None or d < best_d:
            best, best_d = c, d
    return best


def zone_blocks(zone, shape):
    """Blocks of one zone cut with `shape`: (t0, h0, w0, et, eh, ew) in (bt,
    bh, bw) raster order, clipped to the zone's real extent."""
    t0, h0, w0, et, eh, ew = zone
    out = []
    for bt in range(0, et, shape[0]):
        for bh in range(0, eh, shape[1]):
            for bw in range(0, ew, shape[2]):
                out.append((t0 + bt, h0 + bh, w0 + bw, min(shape[0], et - bt),
                            min(shape[1], eh - bh), min(shape[2], ew - bw)))
    return out


def adaptive_layout(T: int, H: int, W: int, zones, shapes):
    """Storage order of the content-adaptive blocks (reading: zones in
    raster order, each zone's blocks in raster order, each block's tokens in
    (t, h, w) raster order, so every block is one contiguous run of tokens).

    Returns (perm, blocks): perm[s] is the raster index (t H + h) W + w of
    the token stored at position s, and blocks the (start, length) of every
    block in storage order."""
    perm, blocks = [], []
    for zone, shape in zip(zones, shapes):
        for (t0, h0, w0, et, eh, ew) in zone_blocks(zone, shape):
            blocks.append((len(perm), et * eh * ew))
            for t in range(t0, t0 + et):
                for h in range(h0, h0 + eh):
                    for w in range(w0, w0 + ew):
                        perm.append((t * H + h) * W + w)
    return np.asarray(perm, np.int64), blocks


def adaptive_plan(v: np.ndarray, a: np.ndarray | None, T: int, H: int, W: int,
                  eps: float = EPS_G):
    """The whole content-adaptive partition of one video ([PRISM] Method 1
    and 2): indicator per zone, volume B(m), shape s*(m), storage order.

    v [N, heads, d] (raster order, N = T H W); a [N] or None.
    Returns dict(zones, g, rho, abar, volumes, shapes, perm, blocks)."""
    v = np.asarray(v, np.float64)
    vg = v.reshape(T, H, W, -1)
    ag = None if a is None else np.asarray(a, np.float64).reshape(T, H, W)
    zones, g, rho, abar = zone_indicators(vg, ag, T, H, W, eps)
    volumes = [block_volume(r) for r in rho]
    shapes = [choose_shape(g[m], volumes[m]) for m in range(len(zones))]
    perm, blocks = adaptive_layout(T, H, W, zones, shapes)
    return dict(zones=zones, g=g, rho=rho, abar=abar, volumes=volumes, shapes=shapes,
                perm=perm, blocks=blocks)


def cross_output_norms(o_video: np.ndarray) -> np.ndarray:
    """a_{t,h,w} = ||h_{t,h,w}||_2: the L2 norm of every video token's A->V
    cross-attention output over all heads and channels ([PRISM] Method 1;
    cached for the next layer).  o_video [B, N, heads, d] -> [B, N]."""
    o = np.asarray(o_video, np.float64)
    return np.sqrt((o.reshape(o.shape[0], o.shape[1], -1) ** 2).sum(axis=2))
