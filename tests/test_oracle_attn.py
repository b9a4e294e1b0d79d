"""Pins for the oracle's attention (CPU only): softmax rows sum to one,
identical keys return mean(V), a single key returns V, a dominant logit
returns its V row, key/value permutation invariance, and agreement with an
explicit-loop textbook softmax (no max subtraction) on tiny inputs."""
import math

import numpy as np
import pytest

import oracle as O


def _r(shape, seed, s=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * s


def test_rows_sum_to_one_via_lse():
    q, k, v = _r((9, 16), 1), _r((23, 16), 2), _r((23, 8), 3)
    scale = 0.25
    o, lse = O.attn(q, k, v, scale)
    s = (q @ k.T) * scale
    assert np.allclose(np.exp(s - lse[:, None]).sum(1), 1.0, atol=1e-13)


def test_identical_keys_give_mean_v():
    q = _r((5, 8), 4)
    k = np.tile(_r((1, 8), 5), (11, 1))
    v = _r((11, 3), 6)
    o, _ = O.attn(q, k, v, 0.3)
    assert np.allclose(o, np.tile(v.mean(0), (5, 1)), atol=1e-13)


def test_single_key_returns_v():
    q, k, v = _r((4, 8), 7), _r((1, 8), 8), _r((1, 5), 9)
    o, lse = O.attn(q, k, v, 1.0)
    assert np.allclose(o, np.tile(v, (4, 1)), atol=1e-14)
    assert np.allclose(lse, (q @ k.T)[:, 0])


def test_dominant_logit_selects_row():
    k = np.eye(6)
    q = np.zeros((1, 6))
    q[0, 4] = 200.0
    v = _r((6, 3), 10)
    o, _ = O.attn(q, k, v, 1.0)
    assert np.allclose(o[0], v[4], atol=1e-12)


def test_key_value_permutation_invariance():
    q, k, v = _r((7, 16), 11), _r((19, 16), 12), _r((19, 16), 13)
    perm = np.random.default_rng(14).permutation(19)
    a, la = O.attn(q, k, v, 0.2)
    b, lb = O.attn(q, k[perm], v[perm], 0.2)
    assert np.allclose(a, b, atol=1e-13) and np.allclose(la, lb, atol=1e-13)


def test_textbook_loops():
    # explicit exp / sum loops, no max subtraction, small magnitudes
    q, k, v = _r((3, 4), 15, 0.5), _r((5, 4), 16, 0.5), _r((5, 2), 17)
    scale = 1 / math.sqrt(4)
    o, lse = O.attn(q, k, v, scale)
    for i in range(3):
        w = []
        for j in range(5):
            dot = 0.0
            for c in range(4):
                dot += q[i, c] * k[j, c]
            w.append(math.exp(dot * scale))
        z = sum(w)
        for c in range(2):
            acc = 0.0
            for j in range(5):
                acc += w[j] * v[j, c]
            assert o[i, c] == pytest.approx(acc / z, rel=1e-12, abs=1e-14)
        assert lse[i] == pytest.approx(math.log(z), rel=1e-12)


def test_bshd_heads_and_batches_are_independent():
    q, k, v = _r((2, 6, 3, 8), 18), _r((2, 6, 3, 8), 19), _r((2, 6, 3, 8), 20)
    o, lse = O.joint_attn(q, k, v, 0.35)
    for b in range(2):
        for h in range(3):
            ob, lb = O.attn(q[b, :, h], k[b, :, h], v[b, :, h], 0.35)
            assert np.allclose(o[b, :, h], ob) and np.allclose(lse[b, :, h], lb)
    # changing another head's K leaves this head's output alone
    k2 = k.copy()
    k2[:, :, 1] += 3.0
    o2, _ = O.joint_attn(q, k2, v, 0.35)
    assert np.array_equal(o2[:, :, 0], o[:, :, 0]) and np.array_equal(o2[:, :, 2], o[:, :, 2])


def test_av_cross_directions():
    qv, kv, vv = _r((1, 12, 2, 8), 21), _r((1, 12, 2, 8), 22), _r((1, 12, 2, 8), 23)
    qa, ka, va = _r((1, 5, 2, 8), 24), _r((1, 5, 2, 8), 25), _r((1, 5, 2, 8), 26)
    ov, oa = O.av_cross_attn(qv, kv, vv, qa, ka, va, 0.3)
    assert ov.shape == qv.shape and oa.shape == qa.shape
    # video queries see only audio keys: video K/V do not change o_video
    ov2, oa2 = O.av_cross_attn(qv, kv * 0 + 1, vv * 0 - 2, qa, ka, va, 0.3)
    assert np.array_equal(ov2, ov)
    # audio queries see only video keys: audio K/V do not change o_audio
    ov3, oa3 = O.av_cross_attn(qv, kv, vv, qa, ka * 5, va + 1, 0.3)
    assert np.array_equal(oa3, oa)
    # swapping the streams swaps the outputs
    ov4, oa4 = O.av_cross_attn(qa, ka, va, qv, kv, vv, 0.3)
    assert np.allclose(ov4, oa) and np.allclose(oa4, ov)
    # o_video rows are convex combinations of audio V rows
    assert np.all(ov <= va.max(axis=1, keepdims=True) + 1e-12)
    assert np.all(ov >= va.min(axis=1, keepdims=True) - 1e-12)


def test_text_cross_closed_forms():
    qv, kt, vt = _r((2, 9, 3, 8), 31), _r((2, 4, 3, 8), 32), _r((2, 4, 3, 8), 33)
    o = O.text_cross_attn(qv, kt, vt, 0.4)
    assert o.shape == qv.shape
    # one text token: every video query returns that token's value row
    o1 = O.text_cross_attn(qv, kt[:, :1], vt[:, :1], 0.4)
    assert np.allclose(o1, np.broadcast_to(vt[:, :1], qv.shape))
    # identical text keys: uniform weights, the mean of the value rows
    ksame = np.broadcast_to(kt[:, :1], kt.shape).copy()
    om = O.text_cross_attn(qv, ksame, vt, 0.4)
    assert np.allclose(om, np.broadcast_to(vt.mean(axis=1, keepdims=True), qv.shape))
    # worked value with two keys: q = a e0, k0 = e0, k1 = 0 -> weights
    # (e^(a s), 1) / (e^(a s) + 1)
    a, s = 2.5, 0.4
    q = np.zeros((1, 1, 1, 8)); q[0, 0, 0, 0] = a
    k = np.zeros((1, 2, 1, 8)); k[0, 0, 0, 0] = 1.0
    v = _r((1, 2, 1, 8), 34)
    w0 = math.exp(a * s) / (math.exp(a * s) + 1.0)
    assert np.allclose(O.text_cross_attn(q, k, v, s)[0, 0, 0], w0 * v[0, 0, 0] + (1 - w0) * v[0, 1, 0])
    # permuting the text tokens (keys with their values) changes nothing
    perm = np.array([2, 0, 3, 1])
    assert np.allclose(O.text_cross_attn(qv, kt[:, perm], vt[:, perm], 0.4), o)
    # heads are independent: another head's text keys do not move this head
    kt2 = kt.copy(); kt2[:, :, 1] *= -3.0
    o2 = O.text_cross_attn(qv, kt2, vt, 0.4)
    assert np.array_equal(o2[:, :, 0], o[:, :, 0]) and np.array_equal(o2[:, :, 2], o[:, :, 2])


def _mask_layout():
    segs = [O.Segment(O.SEG_VIDEO, 2 * 3 * 4, 2, 3, 4, t0=-2), O.Segment(O.SEG_VIDEO, 3 * 3 * 4, 3, 3, 4),
            O.Segment(O.SEG_AUDIO, 7, t_num=21, t_den=218), O.Segment(O.SEG_TEXT, 5)]
    return O.Layout(segs)


def test_masked_rows_follow_positions():
    lay = _mask_layout()
    rng = np.random.default_rng(41)
    mask = (rng.random((2, 5, 3, 4)) < 0.4).astype(np.uint8)
    rows = O.masked_rows(lay, mask)
    pos = O.positions(lay)
    for b in range(2):
        # every masked (frame, h, w) appears exactly once, at the token whose
        # position is (frame - 2, h, w): the first two frames are the
        # conditioning frames at t = -2, -1
        want = sorted((f - 2, h, w) for f, h, w in zip(*np.nonzero(mask[b])))
        got = sorted(tuple(int(x) for x in pos[r]) for r in rows[b])
        assert got == want
        assert np.all(np.diff(rows[b]) > 0)  # sequence order, no repeats
        assert np.all(rows[b] < 60)          # video tokens only (audio/text start at 60)


def test_masked_joint_special_cases():
    lay = _mask_layout()
    n = lay.n_tokens
    q, k, v = _r((2, n, 2, 8), 42), _r((2, n, 2, 8), 43), _r((2, n, 2, 8), 44)
    o0 = _r((2, n, 2, 8), 45)
    full, _ = O.joint_attn(q, k, v, 0.3)
    # all video tokens masked: the video rows are the joint-attention rows and
    # the audio/text rows keep their initial value
    rows = O.masked_rows(lay, np.ones((2, 5, 3, 4), np.uint8))
    o = O.masked_joint_attn(q, k, v, o0, rows, 0.3)
    assert np.allclose(o[:, :60], full[:, :60]) and np.array_equal(o[:, 60:], o0[:, 60:])
    # empty mask: nothing changes
    rows0 = O.masked_rows(lay, np.zeros((2, 5, 3, 4), np.uint8))
    assert np.array_equal(O.masked_joint_attn(q, k, v, o0, rows0, 0.3), o0)
    # a partial mask: masked rows equal those of full joint attention (each
    # row sees every key), the others are untouched
    mask = np.zeros((2, 5, 3, 4), np.uint8)
    mask[0, 1, 2, 3] = 1
    mask[1, 3:, :2, 1:3] = 1
    rows = O.masked_rows(lay, mask)
    o = O.masked_joint_attn(q, k, v, o0, rows, 0.3)
    for b in range(2):
        keep = np.setdiff1d(np.arange(n), rows[b])
        assert np.allclose(o[b, rows[b]], full[b, rows[b]])
        assert np.array_equal(o[b, keep], o0[b, keep])
