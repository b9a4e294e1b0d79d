"""mmdit_av_cross_attn_noalloc: the cross-attention entry point that uses the
library's fixed device scratch array instead of a caller workspace, for
callers that cannot allocate device memory (a plugin inside a runtime that
owns every device allocation, or a serving loop that forbids allocation after
start-up).  Its output must match the workspace entry point's on the same
inputs, on two calls in a row (the shared array keeps the previous call's
contents, which must not leak into the next result).

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test."""
import ctypes as C
import math

import numpy as np
import pytest

from joint_video_audio_rope_b200 import workloads as WL

from _util import BF16_MAX_ABS, BF16_REL_L2, errors, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from joint_video_audio_rope_b200 import build
    build.build()
    from joint_video_audio_rope_b200 import mmdit
    return mmdit


def _inputs(seed, grid=(21, 14, 16), heads=4):
    # 21x14x16 = 4704 video tokens = 37 key tiles: the audio-query direction is
    # split, so the partial results really go through the scratch array
    w = WL.Workload("noalloc", [WL.video(*grid), WL.audio(218)], batch=2, heads=heads,
                    head_dim=128, dtype="bf16", seed=seed, qk_std=WL.INV_SQRT_128,
                    v_std=WL.INV_SQRT_128)
    x = WL.generate(w)
    return w, {n: to_device(x[n], "bf16") for n in ("q", "k", "v")}


def _slices(w, dev, out):
    v0, v1 = w.video_range()
    a0, a1 = w.audio_range()
    return ([dev[n][:, v0:v1] for n in ("q", "k", "v")] + [dev[n][:, a0:a1] for n in ("q", "k", "v")]
            + [out[:, v0:v1], out[:, a0:a1]])


def _run_workspace(M, w, dev):
    out = torch.full_like(dev["q"], float("nan"))
    t = _slices(w, dev, out)
    dv, da = M.desc_of(t[0]), M.desc_of(t[3])
    n = M.av_cross_attn_workspace_size(dv, da)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    M.av_cross_attn(*t, dv, da, 1 / math.sqrt(128), ws, n)
    torch.cuda.synchronize()
    return out


def _run_noalloc(M, w, dev):
    out = torch.full_like(dev["q"], float("nan"))
    t = _slices(w, dev, out)
    dv, da = M.desc_of(t[0]), M.desc_of(t[3])
    stream = torch.cuda.current_stream().cuda_stream
    # straight through the C ABI
    rc = M.raw("mmdit_av_cross_attn_noalloc")(*[x.data_ptr() for x in t], C.byref(dv),
                                               C.byref(da), 1 / math.sqrt(128), stream)
    assert rc == M.OK, M.last_error()
    torch.cuda.synchronize()
    assert M.device_status() == M.OK
    return out


def _compare(got, ref, what):
    v0 = 0
    g = got.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all(), f"{what}: unwritten output"
    max_abs, rel = errors(g, r)
    assert max_abs <= BF16_MAX_ABS and rel <= BF16_REL_L2, f"{what}: {max_abs:.3e} {rel:.3e}"


def test_noalloc_matches_workspace_entry_on_two_calls(M):
    for call, seed in enumerate((31, 32)):
        w, dev = _inputs(seed)
        ref = _run_workspace(M, w, dev)
        got = _run_noalloc(M, w, dev)
        _compare(got, ref, f"call {call + 1}")


def test_noalloc_lowers_the_split_count_to_fit(M):
    # batch 2 x 16 heads x 256 padded audio rows over 12,500 video tokens: the
    # workspace call splits the video keys five ways (one wave of 160 items),
    # whose partial results (~21 MB) exceed the fixed 16 MiB array, so the
    # allocation-free call has to fall back to fewer, longer splits (three)
    w, dev = _inputs(33, grid=(25, 20, 25), heads=16)
    v0, v1 = w.video_range()
    a0, a1 = w.audio_range()
    dv, da = M.desc_of(dev["q"][:, v0:v1]), M.desc_of(dev["q"][:, a0:a1])
    assert M.av_cross_attn_workspace_size(dv, da) > M.NOALLOC_SCRATCH_BYTES
    ref = _run_workspace(M, w, dev)
    got = _run_noalloc(M, w, dev)
    _compare(got, ref, "reduced split")


def test_noalloc_rejects_problems_beyond_the_scratch(M):
    # 2 batch x 64 heads x 512 padded audio rows x 130 floats = 34 MB > 16 MiB
    dv = M.make_desc(2, 4096, 64, 128, M.BF16)
    da = M.make_desc(2, 300, 64, 128, M.BF16)
    fake = [0x10000 + 4096 * i for i in range(8)]
    rc = M.raw("mmdit_av_cross_attn_noalloc")(*fake, C.byref(dv), C.byref(da), 0.088, None)
    assert rc == M.EINVAL
    assert "maximum" in M.last_error()
