"""Pins for the oracle's Prism content-adaptive blocks (Prism guide, Key ideas
and Method sections 1-2): the 16 candidate shapes, the macro-zone partition,
the directional variance sigma^2_d on features that vary along known axes,
the indicator g_d of a zone that varies along one axis only, the volume
thresholds tau_128 = 0.5 and tau_256 = 0.25, the closed form of the optimal
log-edges l*_d (the Lagrange condition of min sum_d g_d (b_d^2 - 1) subject to
prod_d b_d = B, i.e. b*_d proportional to g_d^(-1/2)), hand-worked shape
choices, the storage order, and the cross-attention output norms."""
import itertools
import math

import numpy as np
import pytest

import oracle as O


def test_sixteen_candidate_shapes():
    allc = [c for B in O.VOLUMES for c in O.shape_candidates(B)]
    assert len(allc) == 16 and len(set(allc)) == 16
    assert [len(O.shape_candidates(B)) for B in O.VOLUMES] == [7, 6, 3]
    # every power-of-two triple with edges 2..8 whose product is a volume
    brute = {c for c in itertools.product((1, 2, 4, 8, 16), repeat=3)
             if min(c) >= 2 and max(c) <= 8 and c[0] * c[1] * c[2] in O.VOLUMES}
    assert brute == set(allc)
    assert O.shape_candidates(64)[0] == (2, 4, 8) and (4, 4, 4) in O.shape_candidates(64)
    assert O.shape_candidates(256) == [(4, 8, 8), (8, 4, 8), (8, 8, 4)]


def test_macro_zones_cover_the_volume():
    T, H, W = 21, 68, 120
    zones = O.macro_zones(T, H, W)
    assert len(zones) == 3 * 9 * 15
    assert sum(et * eh * ew for (_, _, _, et, eh, ew) in zones) == T * H * W
    assert sorted({z[3] for z in zones}) == [5, 8]      # 21 = 8 + 8 + 5
    assert sorted({z[4] for z in zones}) == [4, 8]      # 68 = 8 * 8 + 4
    assert {z[5] for z in zones} == {8}                 # 120 = 15 * 8
    seen = np.zeros((T, H, W), int)
    for (t0, h0, w0, et, eh, ew) in zones:
        seen[t0:t0 + et, h0:h0 + eh, w0:w0 + ew] += 1
    assert np.all(seen == 1)


def _grid(f, ext=(8, 8, 8), D=1):
    t, h, w = np.meshgrid(*(np.arange(e, dtype=np.float64) for e in ext), indexing="ij")
    x = np.zeros(ext + (D,))
    for c in range(D):
        x[..., c] = f(t, h, w, c)
    return x


def test_directional_variance_closed_forms():
    # varies along t only: slice means along t are 0..7 (population variance
    # 5.25); along h and w every slice has the same mean
    s = O.directional_variance(_grid(lambda t, h, w, c: t))
    assert np.allclose(s, [5.25, 0.0, 0.0])
    s = O.directional_variance(_grid(lambda t, h, w, c: 2 * t + 3 * w))
    assert np.allclose(s, [4 * 5.25, 0.0, 9 * 5.25])
    # the channel average: (1/D) sum_c
    s = O.directional_variance(_grid(lambda t, h, w, c: (c + 1) * h, D=2))
    assert np.allclose(s, [0.0, (1 + 4) / 2 * 5.25, 0.0])
    # a short zone (5 frames): variance of 0..4 = 2
    s = O.directional_variance(_grid(lambda t, h, w, c: t, ext=(5, 8, 8)))
    assert np.allclose(s, [2.0, 0.0, 0.0])
    assert np.allclose(O.directional_variance(np.ones((8, 8, 8, 3))), 0.0)
    # a checkerboard varies within every slice but no slice mean moves
    s = O.directional_variance(_grid(lambda t, h, w, c: (-1.0) ** (t + h + w)))
    assert np.allclose(s, 0.0)


def test_indicator_of_a_zone_varying_along_one_axis():
    T, H, W = 8, 8, 16  # two zones along w
    v = np.zeros((T, H, W, 4))
    tt = np.arange(T, dtype=np.float64)[:, None, None]
    v[:, :, :8, :] = tt[..., None] * np.ones((1, H, 8, 4))          # zone 0: along t
    v[:, :, 8:, :] = 0.5 * np.arange(H, dtype=np.float64)[None, :, None, None] \
        * np.ones((T, 1, 8, 4))                                     # zone 1: along h, weaker
    zones, g, rho, abar = O.zone_indicators(v, None, T, H, W)
    eps = O.EPS_G
    assert np.allclose(g[0], [1 + eps, eps, eps])
    assert np.allclose(g[1], [eps, 1 + eps, eps])
    # density: zone 0 has the largest total variance (5.25), zone 1 has 0.25 * 5.25
    assert np.allclose(rho, [1.0, 0.25])
    assert np.all(abar == 0)
    # audio norms varying along w in zone 1 only, with that zone the stronger one
    a = np.ones((T, H, W))
    a[:, :, 8:] = 2.0 + np.arange(8)[None, None, :]
    _, g2, _, abar2 = O.zone_indicators(v, a, T, H, W)
    assert np.allclose(abar2, [1.0 / 5.5, 1.0])                    # zone means 1 and 5.5
    assert np.allclose(g2[0], [1 + eps, eps, eps])                 # a is flat in zone 0
    assert np.allclose(g2[1], [eps, 1 + eps, 1 + eps])             # r_v + abar * vhat_a


def test_volume_thresholds():
    assert O.block_volume(1.0) == 64 and O.block_volume(0.5) == 64
    assert O.block_volume(np.nextafter(0.5, 0)) == 128 and O.block_volume(0.25) == 128
    assert O.block_volume(np.nextafter(0.25, 0)) == 256 and O.block_volume(0.0) == 256


@pytest.mark.parametrize("seed", range(8))
def test_optimal_log_edges_closed_form(seed):
    rng = np.random.default_rng(seed)
    g = rng.uniform(1e-3, 2.0, 3)
    for B in O.VOLUMES:
        ls = O.optimal_log_edges(g, B)
        assert abs(ls.sum() - math.log2(B)) < 1e-12              # prod b*_d = B
        # b*_d ~ g_d^(-1/2): differences of log-edges
        for i, j in ((0, 1), (1, 2), (0, 2)):
            assert abs((ls[i] - ls[j]) + 0.5 * math.log2(g[i] / g[j])) < 1e-12
        # Lagrange condition: g_d b_d^2 is the same for every axis
        lam = g * 4.0 ** ls
        assert np.allclose(lam, lam[0], rtol=1e-12)
        # and b* minimises sum g_d (b_d^2 - 1) on prod b_d = B (random moves
        # along the constraint surface never decrease it)
        f = lambda l: float((g * (4.0 ** l - 1)).sum())
        for _ in range(50):
            d = rng.standard_normal(3)
            d -= d.mean()
            assert f(ls + 0.1 * d) >= f(ls) - 1e-9


def test_hand_worked_shape_choices():
    eps = O.EPS_G
    one_axis = np.array([1 + eps, eps, eps])
    # l* = (-4.64, 5.32, 5.32) at B = 64: (2,4,8) and (2,8,4) tie, the first wins
    assert O.choose_shape(one_axis, 64) == (2, 4, 8)
    assert O.choose_shape(one_axis, 128) == (2, 8, 8)
    assert O.choose_shape(one_axis, 256) == (4, 8, 8)
    iso = np.ones(3)
    assert O.choose_shape(iso, 64) == (4, 4, 4)
    assert O.choose_shape(iso, 128) == (4, 4, 8)          # l* = 7/3 each; first of three ties
    # fine along w only
    assert O.choose_shape(np.array([eps, eps, 1 + eps]), 64) == (4, 8, 2)
    # nearest in log2 space by enumeration
    g = np.array([0.3, 0.05, 0.9])
    ls = O.optimal_log_edges(g, 128)
    d = {c: sum((math.log2(c[i]) - ls[i]) ** 2 for i in range(3))
         for c in O.shape_candidates(128)}
    assert O.choose_shape(g, 128) == min(d, key=d.get)


def test_storage_order_is_a_block_partition():
    T, H, W = 11, 10, 16
    zones = O.macro_zones(T, H, W)
    rng = np.random.default_rng(3)
    allc = [c for B in O.VOLUMES for c in O.shape_candidates(B)]
    shapes = [allc[rng.integers(len(allc))] for _ in zones]
    perm, blocks = O.adaptive_layout(T, H, W, zones, shapes)
    N = T * H * W
    assert sorted(perm.tolist()) == list(range(N))
    assert blocks[0][0] == 0 and sum(n for _, n in blocks) == N
    for (s, n), (s2, _) in zip(blocks, blocks[1:]):
        assert s + n == s2
    for (s, n) in blocks:   # every block is a box of tokens, stored in raster order
        idx = perm[s:s + n]
        t, h, w = idx // (H * W), (idx // W) % H, idx % W
        ext = (t.max() - t.min() + 1) * (h.max() - h.min() + 1) * (w.max() - w.min() + 1)
        assert ext == n and np.all(np.diff(idx) > 0)
        assert n <= 256
    # all-(4,4,4) shapes reproduce the 4x4x4 blocks as token sets
    perm4, blocks4 = O.adaptive_layout(16, 8, 8, O.macro_zones(16, 8, 8),
                                       [(4, 4, 4)] * len(O.macro_zones(16, 8, 8)))
    sets = {frozenset(perm4[s:s + n].tolist()) for s, n in blocks4}
    ref = O.video_blocks(16, 8, 8)
    order = O.positions(O.Layout([O.Segment(O.SEG_VIDEO, 16 * 64, 16, 8, 8,
                                            order=O.ORDER_BLOCK444)]))
    raster = (order[:, 0] * 8 + order[:, 1]) * 8 + order[:, 2]
    assert sets == {frozenset(raster[s:s + n].astype(int).tolist()) for s, n in ref}


def test_adaptive_plan_on_a_planted_volume():
    # zone 0 varies strongly along t, zone 1 weakly along w, zone 2 is flat:
    # densities 1, 1/16 and 0 -> volumes 64, 256, 256; zone 0 is cut finely in t
    T, H, W = 8, 8, 24
    v = np.zeros((T * H * W, 2, 4))
    g = np.zeros((T, H, W, 8))
    g[:, :, :8] = np.arange(T, dtype=float)[:, None, None, None]
    g[:, :, 8:16] = 0.25 * np.arange(8, dtype=float)[None, None, :, None]
    v[:] = g.reshape(T * H * W, 2, 4)
    plan = O.adaptive_plan(v, None, T, H, W)
    assert plan["volumes"] == [64, 256, 256]
    assert plan["shapes"][0] == (2, 4, 8)
    assert plan["shapes"][1] == (8, 8, 4)
    assert len(plan["blocks"]) == 8 + 2 + 2


def test_cross_output_norms():
    rng = np.random.default_rng(5)
    o = rng.standard_normal((2, 7, 3, 4))
    n = O.cross_output_norms(o)
    assert n.shape == (2, 7)
    assert np.allclose(n ** 2, sum((o[:, :, h] ** 2).sum(-1) for h in range(3)))
    o2 = np.zeros((1, 1, 2, 4))
    o2[0, 0, 1] = [3, 0, 4, 0]
    assert O.cross_output_norms(o2)[0, 0] == 5.0
