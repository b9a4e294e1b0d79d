"""Benchmark of the joint video/audio attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference]

One step is one pass of the layer's attention hot path over one batch of the
workload: 3D RoPE of Q and K, then (dense workloads) joint self-attention over
the whole sequence or (block-sparse workloads) block selection and sparse
video self-attention -- on the adaptive workload after the content-adaptive
block plan and the move of Q, K, V to its storage order, O moved back after --
then the bidirectional audio<->video cross-attention (on the adaptive
workload with the A->V output norms for the next step's plan).
Inputs are seeded synthetic tensors of the workload's shape, resident in HBM
before timing; they are larger than L2 (126 MB), so no flush is needed.

The headline workload (default: 720p_cond_b2, the largest dense layer that
fits one GPU) gives the line's value; the other workloads (480p, 720p,
1080p_sparse, 1080p_adaptive) follow under "per_config", timed the same way.  The JSON line
reports algorithmic TFLOP/s (4 * Nq * Nkv * d per head for every attention;
for sparse attention only the selected token pairs), video tokens/s, an
end-to-end figure through the same C-ABI calls with pinned host buffers
copied in and results copied out every step (copies overlapped with compute
on two copy streams), the live roofline of the dominant kernel (CUDA events
around its launches) against the sustained bf16 peak when the timed region
lasts a second or more and the burst peak otherwise, SM clocks sampled
during the timed region, and the fp64 oracle timed on a bounded sample on
the host cores (CPU baseline).

``--impl reference`` times the fp64 oracle instead (the reference arm): each
step is a bounded sample of the same workload on the host cores.

Multi-GPU (torchrun, one process per GPU): every rank runs its own copy of
the workload with no collective on the data path (weak scaling); ranks meet
only at the barriers around the timed region and the max-over-ranks time
reduction.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from joint_video_audio_rope_b200 import workloads as WL  # noqa: E402

METRIC = "joint A/V attention TFLOP/s & video tokens/s per layer, % of B200 bf16 TC peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- ranks

def dist_env():
    """(rank, world, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity on one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------- work model

def attn_flops(nq: int, nkv: int, d: int, heads: int, batch: int) -> float:
    return 4.0 * nq * nkv * d * heads * batch


def dense_step_flops(w: WL.Workload) -> dict:
    n, d, H, B = w.n_tokens, w.head_dim, w.heads, w.batch
    nv, na = w.n_video, w.n_audio
    return {"joint": attn_flops(n, n, d, H, B),
            "cross": attn_flops(nv, na, d, H, B) + attn_flops(na, nv, d, H, B)}


# Channels of the video latent that the flow-matching step interpolates (the
# pages leave the latent width open; 16 is taken).
LATENT_CHANNELS = 16

# Workloads timed after the headline one, each reported under "per_config".
PER_CONFIG = ("480p", "720p", "720p_cond_b2", "1080p_sparse", "1080p_adaptive")

# DRAM bytes per launch of the dominant kernel from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), valid only while the kernel
# source is the one that was captured (sha1 of attn_tc.cu + common.cuh).
NCU_TRAFFIC = {
    # ncu, one joint launch of the 720p_cond_b2 layer (1-pass DRAM counters)
    "720p_cond_b2": {"src": "5837f31e28f5a1b5", "bytes": 6218998528},
}


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha1()
    for f in ("attn_tc.cu", "common.cuh"):
        with open(os.path.join(ROOT, "joint_video_audio_rope_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    t = NCU_TRAFFIC.get(workload)
    if t is None or t["src"] != kernel_source_hash():
        return None
    return t["bytes"]


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi SM clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []      # (host arrival time, csv line)
        self.thread = None
        self.window = None   # host-time window of the timed region

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self, window=None) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = self.lines
        if window is not None:
            inside = [l for l in lines if window[0] <= l[0] <= window[1] + 0.1]
            if inside:
                lines = inside
            else:  # timed region shorter than the sampling period: nearest sample
                mid = 0.5 * (window[0] + window[1])
                lines = sorted(lines, key=lambda l: abs(l[0] - mid))[:1]
        for _, line in lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- oracle (CPU)

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_sample(w: WL.Workload, host: dict, rows: int, seed: int = 0):
    """Run the fp64 oracle on a bounded sample of one step: RoPE of every key
    and of `rows` sampled query rows, those rows' joint attention (or, for the
    sparse workload, their block-sparse attention after pooling and selection
    on all blocks), and the cross-attention of `rows` video rows plus every
    audio row.  Returns (seconds, algorithmic flops of the sample)."""
    import oracle as O
    rng = np.random.default_rng(seed)
    lay = O.Layout([O.Segment(s["kind"], s["n_tokens"], s["T"], s["H"], s["W"], s["t0"],
                              s["t_num"], s["t_den"], s["order"]) for s in w.segments])
    d, H = w.head_dim, w.heads
    scale = 1.0 / math.sqrt(d)
    t0 = time.perf_counter()
    flops = 0.0
    pos = O.positions(lay)
    q = WL.as_f64(host["q"][0], w.dtype)
    k = O.rope(WL.as_f64(host["k"][0], w.dtype), pos, w.theta)
    v = WL.as_f64(host["v"][0], w.dtype)
    sel_rows = np.sort(rng.choice(w.n_tokens, size=min(rows, w.n_tokens), replace=False))
    qr = O.rope(q[sel_rows], pos[sel_rows], w.theta)
    v0, v1 = w.video_range()
    a0, a1 = w.audio_range()
    if not w.sparse:
        for h in range(H):
            O.attn(qr[:, h], k[:, h], v[:, h], scale)
        flops += attn_flops(len(sel_rows), w.n_tokens, d, H, 1)
    else:
        seg = w.segments[0]
        blocks = O.video_blocks(seg["T"], seg["H"], seg["W"])
        qfull = O.rope(q[v0:v1], pos[v0:v1], w.theta)
        qb, kb = O.pool(qfull[None], blocks), O.pool(k[None, v0:v1], blocks)
        starts = np.array([s for s, _ in blocks])
        for r in sel_rows[sel_rows < v1]:
            i = int(np.searchsorted(starts, r, side="right") - 1)
            for h in range(H):
                sel = O.select_row(qb[0, h, i], kb[0, h], w.top_k, float(np.float32(w.top_p)), scale)
                kk = np.concatenate([k[blocks[j][0]:blocks[j][0] + blocks[j][1], h] for j in sel])
                vv = np.concatenate([v[blocks[j][0]:blocks[j][0] + blocks[j][1], h] for j in sel])
                O.attn(qr[sel_rows == r][:, h], kk, vv, scale)
                flops += attn_flops(1, len(kk), d, 1, 1)
    # cross-attention: sampled video rows over the audio keys, every audio row
    # over the video keys
    vrows = sel_rows[(sel_rows >= v0) & (sel_rows < v1)]
    if a1 > a0:
        qa = O.rope(q[a0:a1], pos[a0:a1], w.theta)
        for h in range(H):
            O.attn(qr[np.isin(sel_rows, vrows)][:, h], k[a0:a1, h], v[a0:a1, h], scale)
            O.attn(qa[:, h], k[v0:v1, h], v[v0:v1, h], scale)
        flops += attn_flops(len(vrows), a1 - a0, d, H, 1) + attn_flops(a1 - a0, v1 - v0, d, H, 1)
    return time.perf_counter() - t0, flops


def calibrate_rows(w: WL.Workload, host: dict, target_s: float) -> int:
    """Number of sampled query rows whose oracle sample takes about target_s
    (grown geometrically from a small probe until a probe takes at least 0.7 x
    target_s; the fixed cost of rotating every key is part of each probe)."""
    rows = 8
    for _ in range(6):
        dt, _ = oracle_sample(w, host, rows, seed=1)
        if dt >= 0.7 * target_s or rows >= w.n_tokens:
            break
        rows = int(min(w.n_tokens, rows * min(8.0, max(2.0, 0.8 * target_s / max(dt, 1e-3)))))
    return max(8, rows)


def cpu_baseline(w: WL.Workload, host: dict, target_s: float = 15.0) -> dict:
    """Time the oracle as it stands on a bounded sample (about `target_s`)."""
    rows = calibrate_rows(w, host, target_s)
    dt, flops = oracle_sample(w, host, rows, seed=2)
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows} sampled query rows x {w.heads} heads (+ all audio rows for the "
                      f"cross-attention), keys RoPE'd in full; {dt:.1f} s fp64 numpy",
            "seconds": dt}


# ----------------------------------------------------------------- GPU arm

# A timed region at least this long runs the GPU at its power-capped sustained
# clock: a dominant kernel timed inside it is compared with the sustained bf16
# peak, a shorter one (a burst) with the burst peak.
SUSTAINED_REGION_MS = 1000.0


def pick_peak(peaks: dict, region_ms: float):
    """(peak TFLOP/s, name) of the bf16 peak that matches a timed region."""
    if region_ms >= SUSTAINED_REGION_MS:
        key = "bf16_tflops_sustained"
    else:
        key = "bf16_tflops"
    return peaks.get(key) or FALLBACK_PEAKS[key], key


class Layer:
    """Device tensors of one workload and the call sequence of one step:
    RoPE of Q and K in place, then joint attention (dense workloads) or block
    selection + sparse attention (the block-sparse workload), then both
    directions of the audio<->video cross-attention."""

    def __init__(self, M, w, x, dev):
        import torch
        self.M, self.w = M, w
        up = lambda a: (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev))
        self.q, self.k, self.v = up(x["q"]), up(x["k"]), up(x["v"])
        self.o = torch.empty_like(self.q)
        self.oc = torch.empty_like(self.q)  # video and audio slices take the cross outputs
        q = self.q
        self.desc = M.desc_of(q)
        self.lay = M.make_layout(w.segments)
        self.rope = M.rope_params(w.theta, 44, 42, 42)
        self.scale = 1.0 / math.sqrt(w.head_dim)
        self.v0, self.v1 = w.video_range()
        self.a0, self.a1 = w.audio_range()
        v0, v1, a0, a1 = self.v0, self.v1, self.a0, self.a1
        self.dv, self.da = M.desc_of(q[:, v0:v1]), M.desc_of(q[:, a0:a1])
        ws_cross = M.av_cross_attn_workspace_size(self.dv, self.da)
        self.sparse = w.sparse
        self.adaptive = w.adaptive
        ws_sel = ws_sp = 0
        if self.adaptive:
            # Prism content-adaptive blocks: plan from V and the previous
            # step's A->V output norms, Q/K/V moved to the adaptive order,
            # selection and sparse attention over the plan's block table, O
            # moved back to raster order
            seg = next(s for s in w.segments if s["kind"] == WL.SEG_VIDEO)
            self.grid = (seg["T"], seg["H"], seg["W"])
            T, H, W = self.grid
            self.nz, self.nb = M.adaptive_num_zones(T, H, W), M.adaptive_max_blocks(T, H, W)
            self.zones = torch.empty((w.batch, self.nz, 4), dtype=torch.int32, device=dev)
            self.blocks = torch.empty((w.batch, self.nb, 2), dtype=torch.int32, device=dev)
            self.nblk = torch.empty((w.batch,), dtype=torch.int32, device=dev)
            self.norms = torch.zeros((w.batch, v1 - v0), dtype=torch.float32, device=dev)
            # permuted copies with the strides of the video slice of q
            self.perm = [torch.empty_like(q)[:, v0:v1] for _ in range(4)]
            self.idx = torch.empty((w.batch, w.heads, self.nb, self.nb), dtype=torch.int32,
                                   device=dev)
            self.cnt = torch.empty((w.batch, w.heads, self.nb), dtype=torch.int32, device=dev)
            ws_cross = M.av_cross_attn_norms_workspace_size(self.dv, self.da)
            ws_sel = max(M.adaptive_plan_workspace_size(self.dv, T, H, W),
                         M.block_select_table_workspace_size(self.dv, self.nb))
            ws_sp = M.sparse_attn_table_workspace_size(self.dv, self.nb)
        elif self.sparse:
            self.vlay = M.make_layout([s for s in w.segments if s["kind"] == WL.SEG_VIDEO])
            self.nb = M.num_blocks(self.vlay)
            self.idx = torch.empty((w.batch, w.heads, self.nb, self.nb), dtype=torch.int32,
                                   device=dev)
            self.cnt = torch.empty((w.batch, w.heads, self.nb), dtype=torch.int32, device=dev)
            ws_sel = M.block_select_workspace_size(self.dv, self.vlay)
            ws_sp = M.sparse_attn_workspace_size(self.dv, self.vlay, self.nb)
        self.ws = torch.empty(max(ws_cross, ws_sel, ws_sp, 256), dtype=torch.uint8, device=dev)
        # launches of this library's kernels per step: RoPE 1; joint 1, or
        # table + pooling + scores + selection 4 and table + groups + union +
        # schedule + sparse attention 5, or (adaptive) plan 2 + permute 1 +
        # pooling + scores + selection 3 + groups + union + schedule + sparse
        # attention 4 + permute back 1; cross 3 (+1 for the output norms)
        if self.adaptive:
            self.launches = 1 + 2 + 1 + 3 + 4 + 1 + 4
        else:
            self.launches = 1 + (9 if self.sparse else 1) + 3

    def step(self, stream, ev=None):
        M, w = self.M, self.w
        q, k, v, o, oc = self.q, self.k, self.v, self.o, self.oc
        v0, v1, a0, a1 = self.v0, self.v1, self.a0, self.a1
        if ev is not None:
            ev[0].record(stream)
        M.rope_apply(q, k, self.desc, self.lay, self.rope, stream)
        if ev is not None:
            ev[1].record(stream)
        if self.adaptive:
            T, H, W = self.grid
            pq, pk, pv, po = self.perm
            n = self.ws.numel()
            M.adaptive_plan(v[:, v0:v1], self.norms, self.dv, T, H, W, self.zones, self.blocks,
                            self.nblk, self.nb, self.ws, n, stream=stream)
            M.adaptive_permute([q[:, v0:v1], k[:, v0:v1], v[:, v0:v1]], [pq, pk, pv], self.dv, T, H,
                               W, self.zones, stream=stream)
            M.block_select_table(pq, pk, self.dv, self.blocks, self.nblk, self.nb, w.top_k,
                                 w.top_p, self.scale, self.nb, self.idx, self.cnt, self.ws, n,
                                 stream)
            if ev is not None:
                ev[2].record(stream)
            M.sparse_attn_table(pq, pk, pv, po, self.dv, self.blocks, self.nblk, self.nb,
                                self.idx, self.cnt, self.nb, self.scale, self.ws, n, stream)
            M.adaptive_permute([po], [o[:, v0:v1]], self.dv, T, H, W, self.zones, inverse=True,
                               stream=stream)
            if ev is not None:
                ev[3].record(stream)
            # this step's A->V output norms guide the next step's plan (the
            # one-layer lag of the guidance)
            M.av_cross_attn_norms(q[:, v0:v1], k[:, v0:v1], v[:, v0:v1], q[:, a0:a1], k[:, a0:a1],
                                  v[:, a0:a1], oc[:, v0:v1], oc[:, a0:a1], self.dv, self.da,
                                  self.scale, self.norms, self.ws, n, stream)
            if ev is not None:
                ev[4].record(stream)
            return
        if self.sparse:
            M.block_select(q[:, v0:v1], k[:, v0:v1], self.dv, self.vlay, w.top_k, w.top_p,
                           self.scale, self.nb, self.idx, self.cnt, self.ws, self.ws.numel(),
                           stream)
            if ev is not None:
                ev[2].record(stream)
            M.sparse_attn(q[:, v0:v1], k[:, v0:v1], v[:, v0:v1], o[:, v0:v1], self.dv, self.vlay,
                          self.idx, self.cnt, self.nb, self.scale, self.ws, self.ws.numel(),
                          stream)
        else:
            if ev is not None:
                ev[2].record(stream)
            M.joint_attn(q, k, v, o, self.desc, self.lay, self.scale, stream=stream)
        if ev is not None:
            ev[3].record(stream)
        M.av_cross_attn(q[:, v0:v1], k[:, v0:v1], v[:, v0:v1], q[:, a0:a1], k[:, a0:a1],
                        v[:, a0:a1], oc[:, v0:v1], oc[:, a0:a1], self.dv, self.da, self.scale,
                        self.ws, self.ws.numel(), stream)
        if ev is not None:
            ev[4].record(stream)


def selected_pair_flops(w, idx_h, cnt_h, blen=None):
    """Algorithmic flops of block-sparse attention: 4 d per selected
    (query token, key token) pair, summed over every (batch, head, block).
    blen [B, nblocks]: block lengths (default: the 4x4x4 blocks of the grid)."""
    seg = w.segments[0]
    if blen is None:
        nb = idx_h.shape[2]
        one = np.array([_block_len(seg["T"], seg["H"], seg["W"], b) for b in range(nb)], np.int64)
        blen = np.tile(one, (w.batch, 1))
    pairs = 0
    for b in range(w.batch):
        lb = np.asarray(blen[b], np.int64)
        for h in range(w.heads):
            for i in range(len(lb)):
                pairs += lb[i] * lb[idx_h[b, h, i, :cnt_h[b, h, i]]].sum()
    return 4.0 * pairs * w.head_dim


def time_steps(L, args, dev, stream, world, sampler=None, restore=None):
    """Warm up, then time args.steps steps with CUDA events on `stream`
    (barrier + synchronize on both sides, max over ranks).  Returns
    (ms per step, mean ms of each part, host-time window)."""
    import torch
    M = L.M

    def one(ev=None):
        if restore is not None:
            restore()
        L.step(stream, ev)

    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize(dev)
    if M.device_status(stream) != 0:
        raise RuntimeError("device status after warm-up: " + M.last_error())
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    if sampler is not None:
        sampler.start()
        time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    host_t0 = time.time()
    t_start.record(stream)
    for i in range(args.steps):
        one(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    host_t1 = time.time()
    barrier(world, dev)
    if M.device_status(stream) != 0:
        raise RuntimeError("device status after timing: " + M.last_error())
    ms_total = reduce_max(t_start.elapsed_time(t_end), world, dev)
    names = ["rope", "select" if L.sparse else "none", "sparse" if L.sparse else "joint", "cross"]
    part_ms = {name: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs)
               for j, name in enumerate(names) if name != "none"}
    return ms_total / args.steps, part_ms, (host_t0, host_t1)


def time_call(fn, args, dev, stream, world):
    """Mean device ms of `fn` over args.steps back-to-back calls after
    args.warmup untimed ones (CUDA events, max over ranks)."""
    import torch
    for _ in range(args.warmup):
        fn()
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    return reduce_max(e0.elapsed_time(e1), world, dev) / args.steps


def measure_workload(M, w, args, dev, stream, world, peaks, sampler=None):
    """Timed steps of one workload with inputs resident in HBM: step time,
    algorithmic TFLOP/s, video tokens/s and the dominant kernel against the
    bf16 peak that matches the length of the timed region."""
    import torch
    x = WL.generate(w)
    L = Layer(M, w, x, dev)
    restore = None
    if L.sparse:
        # the selected blocks (so the work) depend on the values: every step
        # starts from the generated Q and K (a device copy counted in the step)
        q0, k0 = L.q.clone(), L.k.clone()

        def restore():
            L.q.copy_(q0)
            L.k.copy_(k0)
    ms_step, part_ms, window = time_steps(L, args, dev, stream, world, sampler, restore)
    flops = dense_step_flops(w)
    res = {}
    if L.sparse:
        idx_h, cnt_h = L.idx.cpu().numpy(), L.cnt.cpu().numpy()
        blen = None
        if L.adaptive:
            nblk = L.nblk.cpu().numpy()
            tab = L.blocks.cpu().numpy()
            blen = [tab[b, :nblk[b], 1] for b in range(w.batch)]
            cnt_h = cnt_h[:, :, :int(nblk.max())]
            zs = L.zones.cpu().numpy()[..., 0].ravel()
            res["adaptive"] = {"zones": int(L.nz), "blocks": int(nblk.sum()),
                               "volumes": {"64": int((zs < 7).sum()),
                                           "128": int(((zs >= 7) & (zs < 13)).sum()),
                                           "256": int((zs >= 13).sum())}}
            res["block_density"] = round(float(np.mean([cnt_h[b].mean() / nblk[b]
                                                        for b in range(w.batch)])), 4)
        else:
            res["block_density"] = round(float(cnt_h.mean() / L.nb), 4)
        flops = {"joint": selected_pair_flops(w, idx_h, cnt_h, blen), "cross": flops["cross"]}
        del idx_h
    step_flops = flops["joint"] + flops["cross"]
    dom = "sparse" if L.sparse else "joint"
    region_ms = ms_step * args.steps
    peak, peak_key = pick_peak(peaks, region_ms)
    achieved = flops["joint"] / (part_ms[dom] / 1e3) / 1e12
    res.update({
        "ms_per_step": round(ms_step, 4),
        "tflops": round(step_flops * world / (ms_step / 1e3) / 1e12, 2),
        "video_tokens_per_s": round(w.batch * w.n_video * world / (ms_step / 1e3), 1),
        "parts_ms": {k_: round(v_, 4) for k_, v_ in part_ms.items()},
        "flops_per_step": flops,
        "dominant": {"kernel": "attn_tc_kernel (" + dom + ")", "achieved": round(achieved, 2),
                     "peak": peak, "frac": round(achieved / peak, 4),
                     "peak_source": f"{peak_key} (timed region {region_ms / 1e3:.2f} s)"},
        "cross_frac": round(flops["cross"] / (part_ms["cross"] / 1e3) / 1e12 / peak, 4),
        "step": ("rope+plan+permute+select+sparse+unpermute+cross_norms" if L.adaptive else
                 "rope+select+sparse+cross" if L.sparse else "rope+joint+cross"),
        "launches_per_step": L.launches,
    })
    return res, L, x, window, step_flops


def e2e_overlapped(L, x, args, dev, stream, world, step_flops):
    """End-to-end steps through the same C-ABI calls from pinned host memory:
    every step copies its Q, K, V in and its outputs (joint or sparse O and
    the cross-attention O) out.  Two device sets of tensors alternate, so the
    input copy of step i+1 (one copy stream) and the output copy of step i
    (another) overlap the compute of the next step; the timed region runs from
    the first input copy to the last output copy."""
    import torch
    M, w = L.M, L.w
    pin = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
    hq, hk, hv = pin(x["q"]), pin(x["k"]), pin(x["v"])
    ho = torch.empty(L.o.shape, dtype=L.o.dtype).pin_memory()
    hoc = torch.empty(L.oc.shape, dtype=L.o.dtype).pin_memory()
    sets = [L, Layer(M, w, x, dev)]
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n = max(2, args.steps)  # as many steps as the timed region: fill and drain amortised
    mk = lambda: [torch.cuda.Event() for _ in range(2)]
    ev_in, ev_comp, ev_out = mk(), mk(), mk()

    def h2d(i):
        S = sets[i % 2]
        if i >= 2:
            h2d_s.wait_event(ev_comp[i % 2])  # step i-2 has finished with this set
        with torch.cuda.stream(h2d_s):
            S.q.copy_(hq, non_blocking=True)
            S.k.copy_(hk, non_blocking=True)
            S.v.copy_(hv, non_blocking=True)
        ev_in[i % 2].record(h2d_s)

    def run(n_steps, e0=None):
        if e0 is not None:
            h2d_s.wait_event(e0)
        h2d(0)
        for i in range(n_steps):
            if i + 1 < n_steps:
                h2d(i + 1)
            S = sets[i % 2]
            stream.wait_event(ev_in[i % 2])
            if i >= 2:
                stream.wait_event(ev_out[i % 2])  # outputs of step i-2 are out
            S.step(stream)
            ev_comp[i % 2].record(stream)
            d2h_s.wait_event(ev_comp[i % 2])
            with torch.cuda.stream(d2h_s):
                ho.copy_(S.o, non_blocking=True)
                hoc.copy_(S.oc, non_blocking=True)
            ev_out[i % 2].record(d2h_s)
        for j in range(min(2, n_steps)):
            stream.wait_event(ev_out[(n_steps - 1 - j) % 2])

    run(2)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run(n, e0)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if M.device_status(stream) != 0:
        raise RuntimeError("device status after the end-to-end steps: " + M.last_error())
    ms = reduce_max(e0.elapsed_time(e1), world, dev) / n
    h2d_b = 3 * L.q.numel() * L.q.element_size()
    d2h_b = 2 * L.o.numel() * L.o.element_size()
    sets.pop()
    return {"value": round(step_flops * world / (ms / 1e3) / 1e12, 2), "unit": UNIT,
            "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b, "ms_per_step": round(ms, 3),
            "steps": n, "copy_gbs": round((h2d_b + d2h_b) / (ms / 1e3) / 1e9, 1),
            "note": "pinned host buffers; input copy of step i+1 and output copy of step i "
                    "on two copy streams, overlapping the compute (two device sets)"}


def run_gpu(args) -> int:
    import torch

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    if rank == 0:
        from joint_video_audio_rope_b200 import build
        build.build()
    barrier(world, dev)
    from joint_video_audio_rope_b200 import mmdit as M

    peaks, peak_src = read_peaks()
    stream = torch.cuda.current_stream(dev)
    w = WL.WORKLOADS[args.workload]

    # ---------------------------------------------------------- headline
    sampler = ClockSampler(local)
    head, L, x, window, step_flops = measure_workload(M, w, args, dev, stream, world, peaks,
                                                      sampler)
    time.sleep(0.15)
    clocks = sampler.stop(window)
    v0, v1 = L.v0, L.v1
    q, k, v = L.q, L.k, L.v

    # --------------------------------------------- text cross-attention
    # The reinforced text cross-attention (video queries over the text keys)
    # is a call of its own, outside the step the metric is defined on.
    text_cross_ms = None
    tx0, tx1 = w.text_range()
    if tx1 > tx0:
        o_text = torch.empty_like(q)
        dtx = M.desc_of(k[:, tx0:tx1])
        text_cross_ms = time_call(
            lambda: M.text_cross_attn(q[:, v0:v1], k[:, tx0:tx1], v[:, tx0:tx1], o_text[:, v0:v1],
                                      L.dv, dtx, L.scale, stream), args, dev, stream, world)
        if M.device_status(stream) != 0:
            raise RuntimeError("device status after the text cross-attention: " + M.last_error())
        del o_text

    # ------------------------- mask-guided region-restricted attention
    masked_ms = None
    n_masked_rows = int(np.count_nonzero(x["mask"])) if w.mask else 0  # one entry per video token
    if w.mask and not L.sparse:
        o_mask = torch.empty_like(q)
        mask_dev = torch.from_numpy(x["mask"]).to(dev)
        nmw = M.masked_joint_attn_workspace_size(L.desc, L.lay)
        ws_mask = torch.empty(nmw, dtype=torch.uint8, device=dev)
        masked_ms = time_call(
            lambda: M.masked_joint_attn(q, k, v, o_mask, L.desc, L.lay, L.scale, mask_dev, ws_mask,
                                        nmw, stream), args, dev, stream, world)
        if M.device_status(stream) != 0:
            raise RuntimeError("device status after the masked attention: " + M.last_error())
        del ws_mask, o_mask

    # ------------------------------------------- flow-matching elementwise
    # The noised input / velocity target and the loss term of the video
    # stream's latent (the video token grid x LATENT_CHANNELS values per item),
    # separate calls: at the workload's batch and at a 64-item batch of the
    # same latent (larger than L2, HBM-bound).
    flow = {}
    n_lat = w.n_video * LATENT_CHANNELS
    for label, items in (("workload_batch", w.batch), ("batch64", 64)):
        g = torch.Generator(device=dev).manual_seed(9)
        z0_l, eps_l, v_l = (torch.randn((items, n_lat), generator=g, device=dev,
                                        dtype=torch.float32).to(torch.bfloat16) for _ in range(3))
        t_l = torch.rand(items, generator=g, device=dev)
        zt_l, u_l = torch.empty_like(z0_l), torch.empty_like(z0_l)
        loss_l = torch.empty(items, device=dev)
        nfw = M.flow_loss_workspace_size(items, n_lat)
        ws_l = torch.empty(max(nfw, 256), dtype=torch.uint8, device=dev)
        t_noise = time_call(lambda: M.flow_noise(z0_l, eps_l, t_l, zt_l, u_l, stream), args, dev,
                            stream, world)
        t_loss = time_call(lambda: M.flow_loss(v_l, z0_l, eps_l, loss_l, ws_l, nfw, stream), args,
                           dev, stream, world)
        nbytes = items * n_lat * 2
        flow[label] = {"items": items, "values_per_item": n_lat,
                       "noise_us": round(t_noise * 1e3, 2),
                       "noise_gbs": round(4 * nbytes / (t_noise / 1e3) / 1e9, 1),
                       "loss_us": round(t_loss * 1e3, 2),
                       "loss_gbs": round(3 * nbytes / (t_loss / 1e3) / 1e9, 1)}
        del z0_l, eps_l, v_l, zt_l, u_l, ws_l
    if M.device_status(stream) != 0:
        raise RuntimeError("device status after the flow-matching kernels: " + M.last_error())

    # ---------------------------------------------------------- end to end
    e2e = e2e_overlapped(L, x, args, dev, stream, world, step_flops)
    del L, x, q, k, v
    torch.cuda.empty_cache()

    # ------------------------------------------- the other workloads
    per_config = {}
    if not args.no_per_config:
        for name in PER_CONFIG:
            if name == w.name:
                continue
            r, Lc, xc, _, _ = measure_workload(M, WL.WORKLOADS[name], args, dev, stream, world,
                                               peaks)
            per_config[name] = r
            del Lc, xc
            torch.cuda.empty_cache()

    # ---------------------------------------------------------- report
    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0
    dom = head["dominant"]
    line = {
        "metric": METRIC, "value": head["tflops"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.n_tokens,
                   "video_tokens": w.n_video, "audio_tokens": w.n_audio, "heads": w.heads,
                   "head_dim": w.head_dim, "parallelism": f"replica x{world} (no collective)",
                   "l2": "inputs larger than L2 (no flush needed)", "step": head["step"]},
        "video_tokens_per_s": head["video_tokens_per_s"],
        "frac_of_peak": round(head["tflops"] / world / dom["peak"], 4),
        "parts_ms": head["parts_ms"],
        "flops_per_step": head["flops_per_step"],
        "e2e": e2e,
        "gpu_launches": head.pop("launches_per_step") * args.steps,
        "roofline": {"bound": "tensor", "kernel": dom["kernel"], "achieved": dom["achieved"],
                     "peak": dom["peak"], "unit": "TFLOP/s", "frac": dom["frac"],
                     "traffic": ncu_traffic(w.name),
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "peak_source": f"{dom['peak_source']} of {peak_src}"},
        "cross_frac": head["cross_frac"],
        "clocks": clocks,
    }
    if "block_density" in head:
        line["block_density"] = head["block_density"]
    peak = dom["peak"]
    if text_cross_ms is not None:
        tf = attn_flops(w.n_video, tx1 - tx0, w.head_dim, w.heads, w.batch)
        line["text_cross"] = {"ms": round(text_cross_ms, 4), "flops": tf,
                              "tflops": round(tf / (text_cross_ms / 1e3) / 1e12, 2),
                              "frac": round(tf / (text_cross_ms / 1e3) / 1e12 / peak, 4),
                              "text_tokens": tx1 - tx0, "launches": args.steps,
                              "note": "separate call, not part of the step or its value"}
    if masked_ms is not None:
        n_rows = n_masked_rows
        mf = 4.0 * n_rows * w.n_tokens * w.head_dim * w.heads
        line["masked_joint"] = {"ms": round(masked_ms, 4), "flops": mf,
                                "tflops": round(mf / (masked_ms / 1e3) / 1e12, 2),
                                "frac": round(mf / (masked_ms / 1e3) / 1e12 / peak, 4),
                                "masked_rows": n_rows, "launches": args.steps,
                                "note": "separate call (rows of masked video tokens over every "
                                        "key), not part of the step or its value"}
    hbm = peaks.get("hbm_gbs") or FALLBACK_PEAKS["hbm_gbs"]
    for f_ in flow.values():
        f_["noise_frac_hbm"] = round(f_["noise_gbs"] / hbm, 4)
        f_["loss_frac_hbm"] = round(f_["loss_gbs"] / hbm, 4)
    line["flow_matching"] = dict(flow, note="separate calls on bf16 latents; bytes = 2 reads + 2 "
                                            "writes (noise) or 3 reads (loss) per value")
    if per_config:
        line["per_config"] = per_config
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, WL.generate(w), args.cpu_seconds)
    print(json.dumps(line), flush=True)
    return 0


def _block_len(T, H, W, b):
    nhb, nwb = -(-H // 4), -(-W // 4)
    tb, r = divmod(b, nhb * nwb)
    hb, wb = divmod(r, nwb)
    return min(4, T - 4 * tb) * min(4, H - 4 * hb) * min(4, W - 4 * wb)


# ----------------------------------------------------------------- reference arm

def run_reference(args) -> int:
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    w = WL.WORKLOADS[args.workload]
    x = WL.generate(w)
    cores = blas_threads()
    # calibrate one step to about args.ref_step_seconds of oracle work
    rows = calibrate_rows(w, x, args.ref_step_seconds)
    for i in range(args.warmup):
        oracle_sample(w, x, rows, seed=100 + i)
    tot_s, tot_f = 0.0, 0.0
    for i in range(args.steps):
        s, f = oracle_sample(w, x, rows, seed=1000 + i)
        tot_s += s
        tot_f += f
    value = tot_f / tot_s / 1e12
    sample = (f"{rows} sampled query rows x {w.heads} heads per step (+ all audio rows for the "
              f"cross-attention), fp64 numpy oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.n_tokens,
                   "video_tokens": w.n_video, "audio_tokens": w.n_audio, "heads": w.heads,
                   "head_dim": w.head_dim, "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="720p_cond_b2", choices=sorted(WL.WORKLOADS))
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the headline workload")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-seconds", type=float, default=6.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
