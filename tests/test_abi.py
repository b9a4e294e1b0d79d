"""Boundary tests that need no GPU: the library loads, exports every function
include/mmdit.h declares, and rejects bad arguments with the documented
status before launching anything (no CUDA call is reached)."""
import ctypes as C
import subprocess

import pytest

from joint_video_audio_rope_b200 import build as B

B.build()
from joint_video_audio_rope_b200 import mmdit as M  # noqa: E402

FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def test_exports_every_declared_symbol():
    names = M.header_functions()
    assert "mmdit_joint_attn" in names and len(names) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", M.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if l.strip()}
    for n in names:
        assert n in exported, n
        assert M.raw(n) is not None
    # nothing but the C ABI is exported
    extra = {e for e in exported if e.startswith("mmdit")} - set(names)
    assert not extra, extra


def test_version_and_error_string():
    assert "sm_100a" in M.version()
    assert isinstance(M.last_error(), str)


def _desc(**kw):
    d = dict(batch=1, n_tokens=112, heads=2, head_dim=128, dtype=M.BF16)
    d.update(kw)
    return M.make_desc(**d)


def _layout(n=112):
    return M.make_layout([dict(kind=M.SEG_VIDEO, n_tokens=n, T=n // 16, H=4, W=4)])


def _rope():
    return M.rope_params(10000.0, 44, 42, 42)


def _rc(fn, *args):
    # stream 0 explicitly: no torch CUDA context is needed on a CPU machine
    import inspect
    nparams = len(inspect.signature(fn).parameters)
    kw = {} if len(args) >= nparams else {"stream": 0}
    with pytest.raises(M.MmditError) as e:
        fn(*args, **kw)
    return e.value.status


def test_rope_rejects_bad_arguments():
    assert _rc(M.rope_apply, None, None, _desc(), _layout(), _rope()) == M.EINVAL
    assert _rc(M.rope_apply, FAKE, FAKE, _desc(dtype=7), _layout(), _rope()) == M.EUNSUPPORTED
    assert _rc(M.rope_apply, FAKE, FAKE, _desc(head_dim=64), _layout(), _rope()) == M.EUNSUPPORTED
    assert _rc(M.rope_apply, FAKE, FAKE, _desc(), _layout(96), _rope()) == M.EINVAL
    assert _rc(M.rope_apply, FAKE, FAKE, _desc(), _layout(), M.rope_params(1e4, 44, 42, 40), 0) == M.EINVAL
    assert _rc(M.rope_apply, FAKE, FAKE, _desc(), _layout(), M.rope_params(1e4, 43, 43, 42), 0) == M.EINVAL
    assert _rc(M.rope_apply, FAKE + 8, FAKE, _desc(), _layout(), _rope()) == M.EINVAL
    assert "NULL" in M.last_error() or "align" in M.last_error()


def test_layout_validation():
    bad_kind = M.make_layout([dict(kind=9, n_tokens=112)])
    assert _rc(M.rope_apply, FAKE, None, _desc(), bad_kind, _rope()) == M.EINVAL
    bad_grid = M.make_layout([dict(kind=M.SEG_VIDEO, n_tokens=112, T=7, H=4, W=5)])
    assert _rc(M.rope_apply, FAKE, None, _desc(), bad_grid, _rope()) == M.EINVAL
    bad_audio = M.make_layout([dict(kind=M.SEG_AUDIO, n_tokens=112, t_num=21, t_den=0)])
    assert _rc(M.rope_apply, FAKE, None, _desc(), bad_audio, _rope()) == M.EINVAL
    lay = M.Layout()
    lay.n_seg = 9
    assert _rc(M.rope_apply, FAKE, None, _desc(), lay, _rope()) == M.EINVAL
    assert "n_seg" in M.last_error()


def test_strides_validation():
    d = _desc(stride_tok=100)  # < heads * head_dim
    assert _rc(M.rope_apply, FAKE, None, d, _layout(), _rope()) == M.EINVAL
    d = _desc(stride_tok=260)  # 520 bytes: not a multiple of 16
    assert _rc(M.rope_apply, FAKE, None, d, _layout(), _rope()) == M.EINVAL
    d = _desc(batch=2, stride_batch=256)  # batch items overlap
    assert _rc(M.rope_apply, FAKE, None, d, _layout(), _rope()) == M.EINVAL


def test_joint_attn_validation():
    d = _desc()
    L = _layout()
    assert _rc(M.joint_attn, FAKE, FAKE, FAKE, None, d, L, 0.1) == M.EINVAL
    assert _rc(M.joint_attn, FAKE, FAKE, FAKE, FAKE, d, L, 0.1) == M.EINVAL  # o aliases q
    assert _rc(M.joint_attn, FAKE, FAKE, FAKE, FAKE + 4096, d, L, -1.0) == M.EINVAL
    # the channel-concat mask is shape-checked: B * frames * H * W = 1 * 7 * 4 * 4
    assert _rc(M.joint_attn, FAKE, FAKE, FAKE, FAKE + 4096, d, L, 0.1, None, None,
               FAKE, 111) == M.EINVAL
    assert "mask" in M.last_error()
    f32 = _desc(dtype=M.F32)
    assert _rc(M.joint_attn, FAKE, FAKE, FAKE, FAKE + 4096, f32, L, 0.1, None, _rope(),
               None, 0) == M.EUNSUPPORTED
    assert M.joint_attn_workspace_size(d) == 0


def test_cross_attn_validation_and_workspace():
    v = _desc(n_tokens=1000, heads=24)
    a = _desc(n_tokens=218, heads=24)
    ws = M.av_cross_attn_workspace_size(v, a)
    assert ws > 0 and ws % 256 == 0
    args = [FAKE + 4096 * i for i in range(8)]
    assert _rc(M.av_cross_attn, *args, v, _desc(n_tokens=218, heads=12), 0.1) == M.EINVAL
    assert _rc(M.av_cross_attn, *args, v, a, 0.1, None, 0) == M.EWORKSPACE
    assert _rc(M.av_cross_attn, *args, v, a, 0.1, FAKE, ws - 1) == M.EWORKSPACE
    assert _rc(M.av_cross_attn, *args, v, _desc(n_tokens=0, heads=24), 0.1, FAKE, ws) == M.EINVAL


def _sparse_layout(T=21, H=68, W=120):
    return M.make_layout([dict(kind=M.SEG_VIDEO, n_tokens=T * H * W, T=T, H=H, W=W,
                               order=M.ORDER_BLOCK444)])


def test_block_counts_and_select_validation():
    L = _sparse_layout()
    assert M.num_blocks(L) == 6 * 17 * 30 == 3060
    assert M.num_blocks(_layout()) == 0  # raster: not a block-sparse layout
    d = _desc(n_tokens=171360, heads=24)
    ws = M.block_select_workspace_size(d, L)
    a = lambda n: (n + 255) // 256 * 256
    # block table, its count, pooled Q and K means, fp32 block scores
    assert ws == a(3060 * 8) + a(4) + 2 * a(24 * 3060 * 128 * 4) + a(24 * 3060 * 3060 * 4)
    assert _rc(M.block_select, FAKE, FAKE, d, L, 32, 0.9, 0.088, 3059, FAKE, FAKE, FAKE, ws) == M.EINVAL
    assert "cap" in M.last_error()
    assert _rc(M.block_select, FAKE, FAKE, d, L, 32, 1.5, 0.088, 3060, FAKE, FAKE, FAKE, ws) == M.EINVAL
    assert _rc(M.block_select, FAKE, FAKE, d, L, -1, 0.9, 0.088, 3060, FAKE, FAKE, FAKE, ws) == M.EINVAL
    assert _rc(M.block_select, FAKE, FAKE, d, L, 32, 0.9, 0.088, 3060, FAKE, FAKE, FAKE, ws - 256) == M.EWORKSPACE
    assert _rc(M.block_select, FAKE, FAKE, d, _layout(171360 // 16 * 16), 32, 0.9, 0.088, 3060,
               FAKE, FAKE, FAKE, ws) == M.EINVAL
    huge = _sparse_layout(T=40, H=80, W=80)  # 10*20*20 = 4000 blocks: fine
    assert M.num_blocks(huge) == 4000
    too_many = _sparse_layout(T=40, H=128, W=128)  # 16384 blocks
    dd = _desc(n_tokens=40 * 128 * 128, heads=2)
    assert _rc(M.block_select, FAKE, FAKE, dd, too_many, 32, 0.9, 0.088, 16384, FAKE, FAKE, FAKE,
               1 << 30) == M.EUNSUPPORTED


def test_sparse_attn_validation():
    L = _sparse_layout()
    d = _desc(n_tokens=171360, heads=24)
    ws = M.sparse_attn_workspace_size(d, L, 3060)
    assert ws > 0
    args = [FAKE, FAKE + 4096, FAKE + 8192, FAKE + 12288]
    assert _rc(M.sparse_attn, *args, d, L, FAKE, FAKE, 3000, 0.088, FAKE, ws) == M.EINVAL
    assert _rc(M.sparse_attn, *args, d, L, FAKE, FAKE, 3060, 0.088, FAKE, ws - 1) == M.EWORKSPACE
    assert _rc(M.sparse_attn, *args, d, L, FAKE, FAKE, 3060, 0.088, FAKE + 8, ws) == M.EINVAL


def test_text_cross_validation():
    f = M.raw("mmdit_text_cross_attn")
    dv, dt = _desc(n_tokens=64), _desc(n_tokens=16)
    assert f(None, FAKE, FAKE, FAKE, C.byref(dv), C.byref(dt), 0.1, None) == M.EINVAL
    bad = _desc(n_tokens=16, heads=3)
    assert f(FAKE, FAKE, FAKE, FAKE * 2, C.byref(dv), C.byref(bad), 0.1, None) == M.EINVAL
    empty = _desc(n_tokens=0)
    assert f(FAKE, FAKE, FAKE, FAKE * 2, C.byref(dv), C.byref(empty), 0.1, None) == M.EINVAL
    assert f(FAKE, FAKE, FAKE, FAKE, C.byref(dv), C.byref(dt), 0.1, None) == M.EINVAL  # o is q
    assert f(FAKE, FAKE, FAKE, FAKE * 2, C.byref(dv), C.byref(dt), 0.0, None) == M.EINVAL
    assert f(FAKE + 4, FAKE, FAKE, FAKE * 2, C.byref(dv), C.byref(dt), 0.1, None) == M.EINVAL
    f32 = _desc(n_tokens=16, dtype=M.F32)
    assert f(FAKE, FAKE, FAKE, FAKE * 2, C.byref(dv), C.byref(f32), 0.1, None) == M.EINVAL


def _cond_layout():
    return M.make_layout([dict(kind=M.SEG_VIDEO, n_tokens=32, T=2, H=4, W=4, t0=-2),
                          dict(kind=M.SEG_VIDEO, n_tokens=48, T=3, H=4, W=4),
                          dict(kind=M.SEG_TEXT, n_tokens=32)])


def test_masked_joint_validation_and_workspace():
    f = M.raw("mmdit_masked_joint_attn")
    d, lay = _desc(batch=2), _cond_layout()
    need = M.masked_joint_attn_workspace_size(d, lay)
    # row counts + row lists + compact Q and O rows of all 80 video tokens
    assert need >= 2 * 80 * 2 * 128 * 2 * 2
    ws = 0x100000
    elems = 2 * 5 * 16
    ok = (FAKE, FAKE * 2, FAKE * 3, FAKE * 4, C.byref(d), C.byref(lay), C.c_float(0.1), FAKE * 5)
    assert f(*ok, elems - 1, ws, need, None) == M.EINVAL          # mask size
    assert f(*ok, elems, ws, need - 256, None) == M.EWORKSPACE    # workspace size
    assert f(*ok, elems, ws + 16, need, None) == M.EINVAL         # workspace alignment
    d32 = _desc(batch=2, dtype=M.F32)
    assert f(FAKE, FAKE * 2, FAKE * 3, FAKE * 4, C.byref(d32), C.byref(lay), C.c_float(0.1),
             FAKE * 5, elems, ws, need, None) == M.EUNSUPPORTED
    assert f(FAKE, FAKE * 2, FAKE * 3, FAKE * 2, C.byref(d), C.byref(lay), C.c_float(0.1),
             FAKE * 5, elems, ws, need, None) == M.EINVAL         # o aliases k
    blk = M.make_layout([dict(kind=M.SEG_VIDEO, n_tokens=112, T=7, H=4, W=4,
                              order=M.ORDER_BLOCK444)])
    assert M.masked_joint_attn_workspace_size(_desc(), blk) == 0
    assert f(FAKE, FAKE * 2, FAKE * 3, FAKE * 4, C.byref(_desc()), C.byref(blk), C.c_float(0.1),
             FAKE * 5, 7 * 16, ws, need, None) == M.EUNSUPPORTED


def test_flow_validation_and_workspace():
    noise, loss = M.raw("mmdit_flow_noise"), M.raw("mmdit_flow_loss")
    assert noise(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 100, 104, 7, None) == M.EUNSUPPORTED
    assert noise(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 100, 96, M.BF16, None) == M.EINVAL   # stride < n
    assert noise(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 100, 100, M.BF16, None) == M.EINVAL  # 200 B stride
    assert noise(FAKE, FAKE, FAKE, None, None, 2, 100, 104, M.BF16, None) == M.EINVAL  # no output
    assert noise(FAKE + 2, FAKE, FAKE, FAKE, FAKE, 2, 100, 104, M.BF16, None) == M.EINVAL
    assert noise(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 100, 104, M.BF16, None) == M.EINVAL  # batch 0
    n1, n2 = M.flow_loss_workspace_size(2, 1000), M.flow_loss_workspace_size(2, 10 ** 7)
    assert 0 < n1 <= n2 and n2 % 256 == 0
    assert loss(FAKE, FAKE, FAKE, FAKE, 2, 1000, 1000, M.F32, None, 0, None) == M.EWORKSPACE
    assert loss(FAKE, FAKE, FAKE, FAKE, 2, 1000, 1000, M.F32, 0x100010, n1, None) == M.EINVAL
    assert loss(FAKE, FAKE, None, FAKE, 2, 1000, 1000, M.F32, 0x100000, n1, None) == M.EINVAL


def test_batch_limits_of_row_grids():
    noise = M.raw("mmdit_flow_noise")
    assert noise(FAKE, FAKE, FAKE, FAKE, FAKE, 65536, 100, 104, M.BF16, None) == M.EINVAL
    f = M.raw("mmdit_masked_joint_attn")
    d, lay = _desc(batch=65536), _cond_layout()
    assert f(FAKE, FAKE * 2, FAKE * 3, FAKE * 4, C.byref(d), C.byref(lay), C.c_float(0.1),
             FAKE * 5, 65536 * 80, 0x100000, 1 << 40, None) == M.EINVAL


def test_adaptive_and_table_calls_validate_arguments():
    T, H, W = 21, 68, 120
    assert M.adaptive_num_zones(T, H, W) == 3 * 9 * 15
    assert M.adaptive_max_blocks(T, H, W) == 8 * 405
    assert M.adaptive_num_zones(0, 4, 4) == 0
    d = _desc(n_tokens=T * H * W, heads=24)
    mb = M.adaptive_max_blocks(T, H, W)
    n = M.adaptive_plan_workspace_size(d, T, H, W)
    assert n > 0 and M.adaptive_plan_workspace_size(d, T, H, W - 1) == 0
    plan = lambda *a, **k: _rc(M.adaptive_plan, *a, **k)
    assert plan(FAKE, None, d, T, H, W + 1, FAKE, FAKE, FAKE, mb, FAKE, n) == M.EINVAL
    assert plan(FAKE, None, d, T, H, W, FAKE, FAKE, FAKE, mb - 1, FAKE, n) == M.EINVAL
    assert plan(FAKE, None, d, T, H, W, FAKE, FAKE, FAKE, mb, FAKE, n - 1) == M.EWORKSPACE
    assert plan(FAKE, None, d, T, H, W, FAKE + 8, FAKE, FAKE, mb, FAKE, n) == M.EINVAL  # zones align
    bad = M.adaptive_params(0.2, 0.5, 1e-6)  # tau_256 > tau_128
    assert plan(FAKE, None, d, T, H, W, FAKE, FAKE, FAKE, mb, FAKE, n, bad) == M.EINVAL
    assert plan(FAKE, None, _desc(n_tokens=T * H * W, heads=24, dtype=M.F32), T, H, W, FAKE, FAKE,
                FAKE, mb, FAKE, n) == M.EUNSUPPORTED
    perm = lambda *a: _rc(M.adaptive_permute, *a)
    assert perm([FAKE], [FAKE], d, T, H, W, FAKE) == M.EINVAL             # dst aliases src
    assert perm([FAKE] * 4, [FAKE * 2] * 4, d, T, H, W, FAKE) == M.EINVAL  # at most three
    assert perm([FAKE], [FAKE * 2], d, T, H, W, None) == M.EINVAL
    # block-table selection / sparse attention
    ns = M.block_select_table_workspace_size(d, mb)
    assert ns > 0 and M.block_select_table_workspace_size(d, 7000) == 0
    sel = lambda *a: _rc(M.block_select_table, *a)
    assert sel(FAKE, FAKE, d, FAKE, FAKE, mb, 32, 0.9, 0.088, mb - 1, FAKE, FAKE, FAKE, ns) == M.EINVAL
    assert sel(FAKE, FAKE, d, FAKE, FAKE, 7000, 32, 0.9, 0.088, 7000, FAKE, FAKE, FAKE, ns) == M.EINVAL
    assert sel(FAKE, FAKE, d, None, FAKE, mb, 32, 0.9, 0.088, mb, FAKE, FAKE, FAKE, ns) == M.EINVAL
    assert sel(FAKE, FAKE, d, FAKE, FAKE, mb, 32, 0.9, 0.088, mb, FAKE, FAKE, FAKE, ns - 1) == M.EWORKSPACE
    nsp = M.sparse_attn_table_workspace_size(d, mb)
    assert nsp > 0
    sp = lambda *a: _rc(M.sparse_attn_table, *a)
    args = [FAKE, FAKE + 4096, FAKE + 8192, FAKE + 12288]
    assert sp(*args, d, FAKE, FAKE, mb, FAKE, FAKE, mb - 1, 0.088, FAKE, nsp) == M.EINVAL
    assert sp(*args, d, FAKE + 4, FAKE, mb, FAKE, FAKE, mb, 0.088, FAKE, nsp) == M.EINVAL  # align
    assert sp(*args, d, FAKE, FAKE, mb, FAKE, FAKE, mb, 0.088, FAKE, nsp - 1) == M.EWORKSPACE
    assert sp(FAKE, FAKE, FAKE, FAKE, d, FAKE, FAKE, mb, FAKE, FAKE, mb, 0.088, FAKE, nsp) == M.EINVAL


def test_cross_norms_validation():
    dv, da = _desc(n_tokens=4096), _desc(n_tokens=218)
    n = M.av_cross_attn_norms_workspace_size(dv, da)
    assert n == M.av_cross_attn_workspace_size(dv, da) + (4096 * 2 * 4 + 255) // 256 * 256
    ptrs = [FAKE + 4096 * i for i in range(8)]
    f = lambda *a: _rc(M.av_cross_attn_norms, *a)
    assert f(*ptrs, dv, da, 0.088, None, FAKE, n) == M.EINVAL
    assert f(*ptrs, dv, da, 0.088, FAKE + 2, FAKE, n) == M.EINVAL
    assert f(*ptrs, dv, da, 0.088, FAKE, FAKE, n - 1) == M.EWORKSPACE
    assert f(*ptrs, dv, _desc(n_tokens=218, heads=3), 0.088, FAKE, FAKE, n) == M.EINVAL
