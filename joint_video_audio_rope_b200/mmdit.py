"""Thin ctypes binding of libmmdit.so (the C ABI in include/mmdit.h).

Argument marshalling only: every step of the hot path runs in the library's
sm_100a kernels.  Functions carry the C names without the ``mmdit_`` prefix.
Tensors are torch tensors (PyTorch supplies device memory and streams) or raw
integer device addresses.  A non-zero status raises ``MmditError`` with the
library's thread-local message.  If the shared library is missing this module
raises ImportError: there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os
import re
from typing import Iterable, Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
# MMDIT_LIB may point at another build of the same library (e.g. a variant).
LIB_PATH = os.environ.get("MMDIT_LIB") or os.path.join(_PKG, "libmmdit.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "mmdit.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing; build it with "
                      "`python -m joint_video_audio_rope_b200.build`")
_lib = C.CDLL(LIB_PATH)

OK, EINVAL, EUNSUPPORTED, EWORKSPACE, ECUDA, ETIMEOUT, EDEVCHECK = range(7)
BF16, F32 = 0, 1
SEG_VIDEO, SEG_AUDIO, SEG_TEXT = 0, 1, 2
ORDER_RASTER, ORDER_BLOCK444 = 0, 1
MAX_SEGMENTS = 8


class Segment(C.Structure):
    _fields_ = [(n, C.c_int32) for n in
                ("kind", "n_tokens", "T", "H", "W", "t0", "t_num", "t_den", "order")]


class Layout(C.Structure):
    _fields_ = [("n_seg", C.c_int32), ("seg", Segment * MAX_SEGMENTS)]


class TensorDesc(C.Structure):
    _fields_ = [("batch", C.c_int32), ("n_tokens", C.c_int32), ("heads", C.c_int32),
                ("head_dim", C.c_int32), ("dtype", C.c_int32),
                ("stride_tok", C.c_int64), ("stride_batch", C.c_int64)]


class RopeParams(C.Structure):
    _fields_ = [("theta", C.c_float), ("dim_t", C.c_int32), ("dim_h", C.c_int32),
                ("dim_w", C.c_int32)]


class AdaptiveParams(C.Structure):
    _fields_ = [("tau_128", C.c_float), ("tau_256", C.c_float), ("eps", C.c_float)]


_P = C.c_void_p
_D = C.POINTER(TensorDesc)
_L = C.POINTER(Layout)
_R = C.POINTER(RopeParams)
_SIGS = {
    "mmdit_rope_apply": (C.c_int, [_P, _P, _D, _L, _R, _P]),
    "mmdit_joint_attn": (C.c_int, [_P, _P, _P, _P, _P, _D, _L, C.c_float, _R, _P, C.c_int64,
                                   _P, C.c_size_t, _P]),
    "mmdit_joint_attn_workspace_size": (C.c_size_t, [_D]),
    "mmdit_av_cross_attn": (C.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _D, _D, C.c_float, _P,
                                      C.c_size_t, _P]),
    "mmdit_av_cross_attn_workspace_size": (C.c_size_t, [_D, _D]),
    "mmdit_text_cross_attn": (C.c_int, [_P, _P, _P, _P, _D, _D, C.c_float, _P]),
    "mmdit_masked_joint_attn": (C.c_int, [_P, _P, _P, _P, _D, _L, C.c_float, _P, C.c_int64, _P,
                                          C.c_size_t, _P]),
    "mmdit_masked_joint_attn_workspace_size": (C.c_size_t, [_D, _L]),
    "mmdit_flow_noise": (C.c_int, [_P, _P, _P, _P, _P, C.c_int32, C.c_int64, C.c_int64,
                                   C.c_int32, _P]),
    "mmdit_flow_loss": (C.c_int, [_P, _P, _P, _P, C.c_int32, C.c_int64, C.c_int64, C.c_int32, _P,
                                  C.c_size_t, _P]),
    "mmdit_flow_loss_workspace_size": (C.c_size_t, [C.c_int32, C.c_int64]),
    "mmdit_av_cross_attn_noalloc": (C.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _D, _D, C.c_float,
                                              _P]),
    "mmdit_block_select": (C.c_int, [_P, _P, _D, _L, C.c_int, C.c_float, C.c_float, C.c_int,
                                     _P, _P, _P, C.c_size_t, _P]),
    "mmdit_block_select_workspace_size": (C.c_size_t, [_D, _L]),
    "mmdit_sparse_attn": (C.c_int, [_P, _P, _P, _P, _D, _L, _P, _P, C.c_int, C.c_float, _P,
                                    C.c_size_t, _P]),
    "mmdit_sparse_attn_workspace_size": (C.c_size_t, [_D, _L, C.c_int]),
    "mmdit_num_blocks": (C.c_int, [_L]),
    "mmdit_av_cross_attn_norms": (C.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _D, _D, C.c_float,
                                            _P, _P, C.c_size_t, _P]),
    "mmdit_av_cross_attn_norms_workspace_size": (C.c_size_t, [_D, _D]),
    "mmdit_adaptive_num_zones": (C.c_int, [C.c_int, C.c_int, C.c_int]),
    "mmdit_adaptive_max_blocks": (C.c_int, [C.c_int, C.c_int, C.c_int]),
    "mmdit_adaptive_plan": (C.c_int, [_P, _P, _D, C.c_int, C.c_int, C.c_int,
                                      C.POINTER(AdaptiveParams), _P, _P, _P, C.c_int, _P,
                                      C.c_size_t, _P]),
    "mmdit_adaptive_plan_workspace_size": (C.c_size_t, [_D, C.c_int, C.c_int, C.c_int]),
    "mmdit_adaptive_permute": (C.c_int, [C.POINTER(C.c_void_p), C.POINTER(C.c_void_p), C.c_int,
                                         _D, C.c_int, C.c_int, C.c_int, _P, C.c_int, _P]),
    "mmdit_block_select_table": (C.c_int, [_P, _P, _D, _P, _P, C.c_int, C.c_int, C.c_float,
                                           C.c_float, C.c_int, _P, _P, _P, C.c_size_t, _P]),
    "mmdit_block_select_table_workspace_size": (C.c_size_t, [_D, C.c_int]),
    "mmdit_sparse_attn_table": (C.c_int, [_P, _P, _P, _P, _D, _P, _P, C.c_int, _P, _P, C.c_int,
                                          C.c_float, _P, C.c_size_t, _P]),
    "mmdit_sparse_attn_table_workspace_size": (C.c_size_t, [_D, C.c_int]),
    "mmdit_device_status": (C.c_int, [_P]),
    "mmdit_selftest_wait_timeout": (C.c_int, [C.c_int, _P, _P]),
    "mmdit_last_error": (C.c_char_p, []),
    "mmdit_version": (C.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class MmditError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"mmdit status {status}: {msg}")
        self.status = status


def header_functions() -> list:
    """Names of the functions include/mmdit.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(mmdit_[a-z0-9_]+)\s*\(", text)))


def last_error() -> str:
    return _lib.mmdit_last_error().decode()


def version() -> str:
    return _lib.mmdit_version().decode()


def _check(rc: int) -> int:
    if rc != OK:
        raise MmditError(rc, last_error())
    return rc


# ---------------------------------------------------------------- marshalling

def make_layout(segments: Sequence[dict]) -> Layout:
    lay = Layout()
    lay.n_seg = len(segments)
    for i, s in enumerate(segments):
        seg = lay.seg[i]
        for k in ("kind", "n_tokens", "T", "H", "W", "t0", "t_num", "t_den", "order"):
            setattr(seg, k, int(s.get(k, 1 if k in ("t_num", "t_den") else 0)))
    return lay


def make_desc(batch, n_tokens, heads, head_dim, dtype, stride_tok=None, stride_batch=None):
    st = heads * head_dim if stride_tok is None else stride_tok
    sb = st * n_tokens if stride_batch is None else stride_batch
    return TensorDesc(batch, n_tokens, heads, head_dim, dtype, st, sb)


def desc_of(t) -> TensorDesc:
    """Descriptor of a torch tensor viewed as [B, N, heads, head_dim]."""
    import torch
    if t.dim() != 4 or t.stride(3) != 1 or t.stride(2) != t.shape[3]:
        raise ValueError("expected [B, N, heads, head_dim] with packed heads and channels")
    dt = {torch.bfloat16: BF16, torch.float32: F32}[t.dtype]
    return TensorDesc(t.shape[0], t.shape[1], t.shape[2], t.shape[3], dt, t.stride(1), t.stride(0))


def rope_params(theta: float, dim_t: int, dim_h: int, dim_w: int) -> RopeParams:
    return RopeParams(theta, dim_t, dim_h, dim_w)


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ref(x):
    return None if x is None else C.byref(x)


# ---------------------------------------------------------------- entry points

def rope_apply(q, k, desc: TensorDesc, layout: Layout, rope: RopeParams, stream=None) -> None:
    _check(_lib.mmdit_rope_apply(_ptr(q), _ptr(k), C.byref(desc), C.byref(layout), C.byref(rope),
                                 _stream(stream)))


def joint_attn(q, k, v, o, desc: TensorDesc, layout: Layout, scale: float, lse=None,
               rope_q: Optional[RopeParams] = None, cond_mask=None, mask_elems: int = 0,
               workspace=None, ws_bytes: int = 0, stream=None) -> None:
    _check(_lib.mmdit_joint_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), C.byref(desc),
                                 C.byref(layout), scale, _ref(rope_q), _ptr(cond_mask),
                                 mask_elems, _ptr(workspace), ws_bytes, _stream(stream)))


def joint_attn_workspace_size(desc: TensorDesc) -> int:
    return _lib.mmdit_joint_attn_workspace_size(C.byref(desc))


def av_cross_attn(qv, kv, vv, qa, ka, va, o_video, o_audio, video: TensorDesc,
                  audio: TensorDesc, scale: float, workspace=None, ws_bytes: int = 0,
                  stream=None) -> None:
    _check(_lib.mmdit_av_cross_attn(_ptr(qv), _ptr(kv), _ptr(vv), _ptr(qa), _ptr(ka), _ptr(va),
                                    _ptr(o_video), _ptr(o_audio), C.byref(video), C.byref(audio),
                                    scale, _ptr(workspace), ws_bytes, _stream(stream)))


def av_cross_attn_workspace_size(video: TensorDesc, audio: TensorDesc) -> int:
    return _lib.mmdit_av_cross_attn_workspace_size(C.byref(video), C.byref(audio))


def text_cross_attn(qv, kt, vt, o_video, video: TensorDesc, text: TensorDesc, scale: float,
                    stream=None) -> None:
    """o_video = softmax(qv kt^T * scale) vt: video queries over the text
    keys (the reinforced text cross-attention); no workspace."""
    _check(_lib.mmdit_text_cross_attn(_ptr(qv), _ptr(kt), _ptr(vt), _ptr(o_video), C.byref(video),
                                      C.byref(text), scale, _stream(stream)))


def masked_joint_attn(q, k, v, o, desc: TensorDesc, layout: Layout, scale: float, mask,
                      workspace=None, ws_bytes: int = 0, stream=None) -> None:
    """Joint-attention rows of the video tokens whose uint8 mask [B, F, H, W]
    value is non-zero; every other row of o is left as it was.  Workspace from
    masked_joint_attn_workspace_size."""
    n = 0 if mask is None else mask.numel()
    _check(_lib.mmdit_masked_joint_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), C.byref(desc),
                                        C.byref(layout), scale, _ptr(mask), n, _ptr(workspace),
                                        ws_bytes, _stream(stream)))


def masked_joint_attn_workspace_size(desc: TensorDesc, layout: Layout) -> int:
    return _lib.mmdit_masked_joint_attn_workspace_size(C.byref(desc), C.byref(layout))


def _items(x):
    """(batch, n, stride, dtype) of a [B, ...] tensor whose items are contiguous
    runs (the trailing dimensions of each item packed)."""
    import torch
    b = x.shape[0]
    n = x[0].numel() if b else 0
    dt = {torch.bfloat16: BF16, torch.float32: F32}[x.dtype]
    return b, n, (x.stride(0) if b else n), dt


def flow_noise(z0, eps, t, zt=None, u=None, stream=None) -> None:
    """zt = t z0 + (1 - t) eps and u = z0 - eps per batch item (t: float
    [B] on the device); [B, ...] tensors whose items are contiguous runs."""
    b, n, st, dt = _items(z0)
    _check(_lib.mmdit_flow_noise(_ptr(z0), _ptr(eps), _ptr(t), _ptr(zt), _ptr(u), b, n, st, dt,
                                 _stream(stream)))


def flow_loss_workspace_size(batch: int, n: int) -> int:
    return _lib.mmdit_flow_loss_workspace_size(batch, n)


def flow_loss(v, z0, eps, loss, workspace=None, ws_bytes: int = 0, stream=None) -> None:
    """loss[b] = sum over item b of (v - (z0 - eps))^2, fp32, fixed summation
    order.  Workspace from flow_loss_workspace_size."""
    b, n, st, dt = _items(z0)
    _check(_lib.mmdit_flow_loss(_ptr(v), _ptr(z0), _ptr(eps), _ptr(loss), b, n, st, dt,
                                _ptr(workspace), ws_bytes, _stream(stream)))


NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024  # MMDIT_NOALLOC_SCRATCH_BYTES


def av_cross_attn_noalloc(qv, kv, vv, qa, ka, va, o_video, o_audio, video: TensorDesc,
                          audio: TensorDesc, scale: float, stream=None) -> None:
    """av_cross_attn without a workspace: the library's fixed device scratch
    array is used instead (for callers that cannot allocate device memory)."""
    _check(_lib.mmdit_av_cross_attn_noalloc(_ptr(qv), _ptr(kv), _ptr(vv), _ptr(qa), _ptr(ka),
                                            _ptr(va), _ptr(o_video), _ptr(o_audio),
                                            C.byref(video), C.byref(audio), scale,
                                            _stream(stream)))


def block_select(q, k, desc: TensorDesc, layout: Layout, top_k: int, top_p: float, scale: float,
                 cap: int, block_idx, block_cnt, workspace=None, ws_bytes: int = 0,
                 stream=None) -> None:
    _check(_lib.mmdit_block_select(_ptr(q), _ptr(k), C.byref(desc), C.byref(layout), top_k, top_p,
                                   scale, cap, _ptr(block_idx), _ptr(block_cnt), _ptr(workspace),
                                   ws_bytes, _stream(stream)))


def block_select_workspace_size(desc: TensorDesc, layout: Layout) -> int:
    return _lib.mmdit_block_select_workspace_size(C.byref(desc), C.byref(layout))


def sparse_attn(q, k, v, o, desc: TensorDesc, layout: Layout, block_idx, block_cnt, cap: int,
                scale: float, workspace=None, ws_bytes: int = 0, stream=None) -> None:
    _check(_lib.mmdit_sparse_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), C.byref(desc),
                                  C.byref(layout), _ptr(block_idx), _ptr(block_cnt), cap, scale,
                                  _ptr(workspace), ws_bytes, _stream(stream)))


def sparse_attn_workspace_size(desc: TensorDesc, layout: Layout, cap: int) -> int:
    return _lib.mmdit_sparse_attn_workspace_size(C.byref(desc), C.byref(layout), cap)


def av_cross_attn_norms(qv, kv, vv, qa, ka, va, o_video, o_audio, video: TensorDesc,
                        audio: TensorDesc, scale: float, video_norm, workspace=None,
                        ws_bytes: int = 0, stream=None) -> None:
    """av_cross_attn plus video_norm[b, n] = ||o_video[b, n]||_2 over all heads
    (float [B, N_video]); workspace from av_cross_attn_norms_workspace_size."""
    _check(_lib.mmdit_av_cross_attn_norms(_ptr(qv), _ptr(kv), _ptr(vv), _ptr(qa), _ptr(ka),
                                          _ptr(va), _ptr(o_video), _ptr(o_audio), C.byref(video),
                                          C.byref(audio), scale, _ptr(video_norm),
                                          _ptr(workspace), ws_bytes, _stream(stream)))


def av_cross_attn_norms_workspace_size(video: TensorDesc, audio: TensorDesc) -> int:
    return _lib.mmdit_av_cross_attn_norms_workspace_size(C.byref(video), C.byref(audio))


def adaptive_params(tau_128: float = 0.5, tau_256: float = 0.25, eps: float = 1e-6):
    return AdaptiveParams(tau_128, tau_256, eps)


def adaptive_num_zones(T: int, H: int, W: int) -> int:
    return _lib.mmdit_adaptive_num_zones(T, H, W)


def adaptive_max_blocks(T: int, H: int, W: int) -> int:
    return _lib.mmdit_adaptive_max_blocks(T, H, W)


def adaptive_plan_workspace_size(desc: TensorDesc, T: int, H: int, W: int) -> int:
    return _lib.mmdit_adaptive_plan_workspace_size(C.byref(desc), T, H, W)


def adaptive_plan(v, a_norm, desc: TensorDesc, T: int, H: int, W: int, zones, blocks, n_blocks,
                  max_blocks: int, workspace=None, ws_bytes: int = 0,
                  params: Optional[AdaptiveParams] = None, stream=None) -> None:
    """Content-adaptive blocks of a raster video: zones int32 [B, n_zones, 4],
    blocks int32 [B, max_blocks, 2], n_blocks int32 [B] (device)."""
    _check(_lib.mmdit_adaptive_plan(_ptr(v), _ptr(a_norm), C.byref(desc), T, H, W, _ref(params),
                                    _ptr(zones), _ptr(blocks), _ptr(n_blocks), max_blocks,
                                    _ptr(workspace), ws_bytes, _stream(stream)))


def adaptive_permute(srcs, dsts, desc: TensorDesc, T: int, H: int, W: int, zones,
                     inverse: bool = False, stream=None) -> None:
    """Raster -> adaptive storage order (inverse: back) of 1..3 tensors."""
    n = len(srcs)
    m = max(n, len(dsts), 1)
    src = (C.c_void_p * m)(*[_ptr(x) for x in srcs])
    dst = (C.c_void_p * m)(*[_ptr(x) for x in dsts])
    _check(_lib.mmdit_adaptive_permute(src, dst, n, C.byref(desc), T, H, W, _ptr(zones),
                                       1 if inverse else 0, _stream(stream)))


def block_select_table(q, k, desc: TensorDesc, blocks, n_blocks, max_blocks: int, top_k: int,
                       top_p: float, scale: float, cap: int, block_idx, block_cnt, workspace=None,
                       ws_bytes: int = 0, stream=None) -> None:
    _check(_lib.mmdit_block_select_table(_ptr(q), _ptr(k), C.byref(desc), _ptr(blocks),
                                         _ptr(n_blocks), max_blocks, top_k, top_p, scale, cap,
                                         _ptr(block_idx), _ptr(block_cnt), _ptr(workspace),
                                         ws_bytes, _stream(stream)))


def block_select_table_workspace_size(desc: TensorDesc, max_blocks: int) -> int:
    return _lib.mmdit_block_select_table_workspace_size(C.byref(desc), max_blocks)


def sparse_attn_table(q, k, v, o, desc: TensorDesc, blocks, n_blocks, max_blocks: int, block_idx,
                      block_cnt, cap: int, scale: float, workspace=None, ws_bytes: int = 0,
                      stream=None) -> None:
    _check(_lib.mmdit_sparse_attn_table(_ptr(q), _ptr(k), _ptr(v), _ptr(o), C.byref(desc),
                                        _ptr(blocks), _ptr(n_blocks), max_blocks, _ptr(block_idx),
                                        _ptr(block_cnt), cap, scale, _ptr(workspace), ws_bytes,
                                        _stream(stream)))


def sparse_attn_table_workspace_size(desc: TensorDesc, max_blocks: int) -> int:
    return _lib.mmdit_sparse_attn_table_workspace_size(C.byref(desc), max_blocks)


def num_blocks(layout: Layout) -> int:
    return _lib.mmdit_num_blocks(C.byref(layout))


def device_status(stream=None) -> int:
    return _lib.mmdit_device_status(_stream(stream))


def selftest_wait_timeout(limit_ms: int, waited_out, stream=None) -> None:
    _check(_lib.mmdit_selftest_wait_timeout(limit_ms, _ptr(waited_out), _stream(stream)))


def raw(name: str):
    """The raw ctypes function of C symbol `name` (for boundary tests)."""
    return getattr(_lib, name)
