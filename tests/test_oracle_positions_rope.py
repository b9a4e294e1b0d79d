"""Pins for the oracle's positions and 3D RoPE (CPU only).

Each test checks the oracle against something other than itself: worked
values from the sources, closed forms computed by hand, or invariants that a
rotation must satisfy (norm preservation, dependence on the position offset
only, identity at position 0)."""
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _layout(*segs):
    return O.Layout(list(segs))


# ---------------------------------------------------------------- positions

def test_audio_positions_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "audio_positions.txt"))
            if l.strip() and not l.startswith("#")]
    pos = O.positions(_layout(O.Segment(O.SEG_AUDIO, 219, t_num=21, t_den=218)))
    for j, num, den in rows:
        assert pos[int(j), 0] == pytest.approx(int(num) / int(den), abs=1e-12)
        assert pos[int(j), 1] == 0 and pos[int(j), 2] == 0
    # exact end points stated by the sources
    assert pos[218, 0] == 21.0 and pos[109, 0] == 10.5 and pos[0, 0] == 0.0


def test_raster_positions_hand_values():
    # 2 frames of a 2x3 grid starting at t=5
    pos = O.positions(_layout(O.Segment(O.SEG_VIDEO, 12, T=2, H=2, W=3, t0=5)))
    expect = [(5, 0, 0), (5, 0, 1), (5, 0, 2), (5, 1, 0), (5, 1, 1), (5, 1, 2),
              (6, 0, 0), (6, 0, 1), (6, 0, 2), (6, 1, 0), (6, 1, 1), (6, 1, 2)]
    assert pos.tolist() == [list(map(float, e)) for e in expect]


def test_cond_frames_negative_time_and_order():
    lay = _layout(O.Segment(O.SEG_VIDEO, 16, T=1, H=4, W=4, t0=-1),
                  O.Segment(O.SEG_VIDEO, 48, T=3, H=4, W=4, t0=0),
                  O.Segment(O.SEG_AUDIO, 32, t_num=21, t_den=218),
                  O.Segment(O.SEG_TEXT, 16))
    pos = O.positions(lay)
    assert pos.shape == (112, 3)
    assert np.all(pos[:16, 0] == -1)                 # conditioning frame: t < 0
    assert np.all(pos[16:64, 0] >= 0)
    assert pos[63].tolist() == [2.0, 3.0, 3.0]
    assert pos[64 + 31, 0] == pytest.approx(651 / 218)
    assert np.all(pos[96:] == 0)                     # text at the origin


def test_block_major_hand_values():
    # T=5, H=4, W=8: blocks (tb,hb,wb) = (0,0,0) (0,0,1) (1,0,0) (1,0,1);
    # the t-slab tb=1 holds one frame, so its blocks are 1x4x4 = 16 tokens.
    pos = O.positions(_layout(O.Segment(O.SEG_VIDEO, 160, T=5, H=4, W=8,
                                        order=O.ORDER_BLOCK444)))
    assert pos[0].tolist() == [0, 0, 0]
    assert pos[1].tolist() == [0, 0, 1]
    assert pos[3].tolist() == [0, 0, 3]
    assert pos[4].tolist() == [0, 1, 0]
    assert pos[16].tolist() == [1, 0, 0]
    assert pos[63].tolist() == [3, 3, 3]
    assert pos[64].tolist() == [0, 0, 4]             # second block, w offset 4
    assert pos[127].tolist() == [3, 3, 7]
    assert pos[128].tolist() == [4, 0, 0]            # short slab, first block
    assert pos[143].tolist() == [4, 3, 3]
    assert pos[144].tolist() == [4, 0, 4]
    assert pos[159].tolist() == [4, 3, 7]
    assert O.video_blocks(5, 4, 8) == [(0, 64), (64, 64), (128, 16), (144, 16)]


@pytest.mark.parametrize("T,H,W", [(5, 6, 9), (21, 8, 12), (4, 4, 4), (1, 3, 5)])
def test_block_major_is_permutation_of_grid(T, H, W):
    pos = O.positions(_layout(O.Segment(O.SEG_VIDEO, T * H * W, T=T, H=H, W=W,
                                        order=O.ORDER_BLOCK444))).astype(int)
    seen = {tuple(p) for p in pos}
    assert len(seen) == T * H * W
    assert seen == {(t, h, w) for t in range(T) for h in range(H) for w in range(W)}
    # every block is contiguous and lies inside one 4x4x4 cube
    for s, n in O.video_blocks(T, H, W):
        cube = {tuple(p // 4) for p in pos[s:s + n]}
        assert len(cube) == 1
    assert sum(n for _, n in O.video_blocks(T, H, W)) == T * H * W


# --------------------------------------------------------------------- rope

def test_rope_bands():
    assert O.rope_bands(128) == (44, 42, 42)
    assert O.rope_bands(64) == (24, 20, 20)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("d", [64, 128])
def test_rope_identity_at_origin(d):
    x = _rand((7, 3, d), 1)
    y = O.rope(x, np.zeros((7, 3)))
    assert np.array_equal(x, y)


@pytest.mark.parametrize("d", [64, 128])
def test_rope_preserves_pair_norms(d):
    x = _rand((9, 2, d), 2)
    pos = np.random.default_rng(3).uniform(-5, 130, (9, 3))
    y = O.rope(x, pos)
    nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    assert np.allclose(nx, ny, rtol=1e-12, atol=1e-12)
    assert np.allclose(np.linalg.norm(x, axis=-1), np.linalg.norm(y, axis=-1), rtol=1e-12)


@pytest.mark.parametrize("d", [64, 128])
def test_rope_dot_depends_only_on_offset(d):
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 1, d))
    k = rng.standard_normal((1, 1, d))
    for _ in range(10):
        p = rng.uniform(-3, 40, (1, 3))
        pk = rng.uniform(-3, 40, (1, 3))
        delta = rng.uniform(-7.5, 7.5, (1, 3))      # fractional and negative
        delta[0, 0] = 21 / 218 * rng.integers(-218, 218)  # audio-like t shift
        a = np.sum(O.rope(q, p) * O.rope(k, pk))
        b = np.sum(O.rope(q, p + delta) * O.rope(k, pk + delta))
        assert a == pytest.approx(b, rel=1e-10, abs=1e-10)


def test_rope_matches_rotation_matrix():
    # Independently built block-diagonal rotation: one explicit 2x2 matrix
    # per channel pair, angle = position of the pair's axis times the pair's
    # frequency, frequencies listed by hand-derivable closed forms below.
    d = 64
    bands = (24, 20, 20)
    freqs = []
    for axis, db in enumerate(bands):
        for i in range(db // 2):
            freqs.append((axis, 10000.0 ** (-(2 * i) / db)))
    rng = np.random.default_rng(5)
    x = rng.standard_normal(d)
    pos = np.array([-1.0, 2.0, 3.0])
    R = np.zeros((d, d))
    for m, (axis, w) in enumerate(freqs):
        a = pos[axis] * w
        R[2 * m:2 * m + 2, 2 * m:2 * m + 2] = [[math.cos(a), -math.sin(a)],
                                               [math.sin(a), math.cos(a)]]
    y = O.rope(x[None, None, :], pos[None, :])[0, 0]
    assert np.allclose(R @ x, y, atol=1e-13)


def test_rope_frequency_worked_values():
    # d=128: bands t/h/w = 44/42/42 channels, theta = 10000.
    # Pair 11 of the t band has frequency 10000^(-22/44) = 1/100, so t = 50*pi
    # turns it by pi/2: (1, 0) -> (0, 1).
    x = np.zeros((1, 1, 128))
    x[0, 0, 22] = 1.0
    y = O.rope(x, np.array([[50 * math.pi, 0.0, 0.0]]))
    assert y[0, 0, 22] == pytest.approx(0.0, abs=1e-12)
    assert y[0, 0, 23] == pytest.approx(1.0, abs=1e-12)
    # Pair 7 of the h band (channels 44+14, 44+15) has frequency
    # 10000^(-14/42) = 10000^(-1/3) = 1/21.5443469...; h = pi*21.5443469...
    # turns it by pi: (1, 0) -> (-1, 0).  Other axes leave it alone.
    x = np.zeros((1, 1, 128))
    x[0, 0, 58] = 1.0
    y = O.rope(x, np.array([[123.0, math.pi * 21.544346900318843, 77.0]]))
    assert y[0, 0, 58] == pytest.approx(-1.0, abs=1e-12)
    assert y[0, 0, 59] == pytest.approx(0.0, abs=1e-12)
    # Pair 0 of the w band (channels 86, 87) turns by exactly w radians.
    x = np.zeros((1, 1, 128))
    x[0, 0, 86] = 1.0
    y = O.rope(x, np.array([[5.0, 9.0, 0.5]]))
    assert y[0, 0, 86] == pytest.approx(math.cos(0.5), abs=1e-14)
    assert y[0, 0, 87] == pytest.approx(math.sin(0.5), abs=1e-14)


def test_rope_band_isolation():
    # moving one axis only changes the channels of that axis' band
    rng = np.random.default_rng(6)
    x = rng.standard_normal((1, 1, 128))
    base = O.rope(x, np.array([[1.0, 2.0, 3.0]]))
    for axis, (lo, hi) in enumerate([(0, 44), (44, 86), (86, 128)]):
        p = np.array([[1.0, 2.0, 3.0]])
        p[0, axis] += 0.7
        y = O.rope(x, p)
        changed = np.nonzero(np.abs(y - base)[0, 0] > 1e-12)[0]
        assert changed.min() >= lo and changed.max() < hi
