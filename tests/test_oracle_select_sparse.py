"""Pins for the oracle's block pooling, hybrid top-k/top-p selection and
block-sparse attention (CPU only): the hand-worked selection fixture, brute
force over all subsets on tiny rows, closed-form block means, and the
reductions of sparse attention to dense attention."""
import itertools
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _scores_from_probs(P, scale):
    """qbar/kbar whose block softmax is exactly P (up to rounding)."""
    n = len(P)
    qbar = np.zeros(4)
    qbar[0] = 1.0
    kbar = np.zeros((n, 4))
    kbar[:, 0] = np.log(P) / scale
    return qbar, kbar


def test_selection_golden():
    for line in open(os.path.join(GOLDEN, "hybrid_selection.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        probs, k, p, expect = [f.strip() for f in line.split("|")]
        P = np.array([float(x) for x in probs.split()])
        qbar, kbar = _scores_from_probs(P, 0.125)
        sel = O.select_row(qbar, kbar, int(k), float(p), 0.125)
        assert sel.tolist() == [int(x) for x in expect.split()]


def _brute_force(P, k, p):
    """Smallest-size subset with mass >= p (largest mass among those), union
    top-k, by enumerating every subset."""
    n = len(P)
    order = sorted(range(n), key=lambda j: (-P[j], j))
    topk = set(order[:min(k, n)])
    best = None
    for size in range(1, n + 1):
        cands = [c for c in itertools.combinations(range(n), size)
                 if sum(P[j] for j in c) >= p]
        if cands:
            best_mass = max(sum(P[j] for j in c) for c in cands)
            best = [set(c) for c in cands if sum(P[j] for j in c) == best_mass]
            break
    if best is None:
        best = [set(range(n))]
    return [sorted(topk | b) for b in best]


@pytest.mark.parametrize("seed", range(12))
def test_selection_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(2, 9))
    qbar = rng.standard_normal(8)
    kbar = rng.standard_normal((n, 8))
    scale = 1 / math.sqrt(8)
    P = O.block_probs(qbar, kbar, scale)
    for k in (0, 1, 2, n):
        for p in (0.1, 0.5, 0.9, 0.99):
            sel = O.select_row(qbar, kbar, k, p, scale).tolist()
            assert sel in _brute_force(P, k, p)
            assert len(sel) >= min(k, n)
            assert sel == sorted(set(sel))


@pytest.mark.parametrize("seed", range(6))
def test_selection_rows_brute_force(seed):
    """select_rows (array steps, every row of a head at once) against brute
    force on tiny rows, including exactly tied scores."""
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(2, 8))
    qbar = rng.standard_normal((5, 8))
    kbar = rng.standard_normal((n, 8))
    if seed % 2:
        kbar[1] = kbar[0]  # two key blocks with identical scores in every row
    scale = 1 / math.sqrt(8)
    for k in (0, 1, 3, n):
        for p in (0.1, 0.5, 0.9, 0.99, 1.0):
            sel = O.select_rows(qbar, kbar, k, p, scale)
            for i in range(5):
                P = O.block_probs(qbar[i], kbar, scale)
                assert sel[i].tolist() in _brute_force(P, k, p)
                if seed % 2:  # ties resolve to the lower id
                    assert not (1 in sel[i] and 0 not in sel[i])


def test_select_from_probs_golden_and_brute_force():
    for line in open(os.path.join(GOLDEN, "hybrid_selection.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        probs, k, p, expect = [f.strip() for f in line.split("|")]
        P = np.array([float(x) for x in probs.split()])
        assert O.select_from_probs(P, int(k), float(p)).tolist() == \
            [int(x) for x in expect.split()]
    rng = np.random.default_rng(7)
    for _ in range(20):
        n = int(rng.integers(2, 9))
        P = rng.dirichlet(np.ones(n))
        for k in (0, 2):
            for p in (0.3, 0.8):
                assert O.select_from_probs(P, k, p).tolist() in _brute_force(P, k, p)


def test_selection_degenerate_cases():
    rng = np.random.default_rng(1)
    qbar, kbar = rng.standard_normal(16), rng.standard_normal((37, 16))
    assert O.select_row(qbar, kbar, 0, 1.0, 0.25).tolist() == list(range(37))
    assert O.select_row(qbar, kbar, 37, 0.0, 0.25).tolist() == list(range(37))
    assert O.select_row(qbar, kbar, 99, 0.5, 0.25).tolist() == list(range(37))
    # p below the top probability: the top-p set is the single best block
    P = O.block_probs(qbar, kbar, 0.25)
    assert O.select_row(qbar, kbar, 0, P.max() * 0.5, 0.25).tolist() == [int(np.argmax(P))]
    # all scores equal: ties resolve to the lowest block ids
    flat = np.zeros((10, 16))
    assert O.select_row(qbar, flat, 3, 0.05, 0.25).tolist() == [0, 1, 2]
    assert O.select_row(qbar, flat, 1, 0.35, 0.25).tolist() == [0, 1, 2, 3]


def test_pool_closed_form():
    T, H, W = 5, 4, 8
    blocks = O.video_blocks(T, H, W)
    N = T * H * W
    x = np.zeros((1, N, 1, 2))
    for s, n in blocks:
        x[0, s:s + n, 0, 0] = np.arange(n)        # in-block index
        x[0, s:s + n, 0, 1] = 7.0                  # constant
    pb = O.pool(x, blocks)
    assert pb.shape == (1, 1, 4, 2)
    assert pb[0, 0, :, 0].tolist() == [31.5, 31.5, 7.5, 7.5]   # (n-1)/2, n=64,64,16,16
    assert np.all(pb[0, 0, :, 1] == 7.0)
    # mean time coordinate: slab 0 holds t=0..3 -> 1.5; the short slab t=4 -> 4
    pos = O.positions(O.Layout([O.Segment(O.SEG_VIDEO, N, T=T, H=H, W=W,
                                          order=O.ORDER_BLOCK444)]))
    pt = O.pool(pos[None, :, None, :], blocks)
    assert pt[0, 0, :, 0].tolist() == [1.5, 1.5, 4.0, 4.0]
    assert pt[0, 0, :, 2].tolist() == [1.5, 5.5, 1.5, 5.5]


def _sparse_case(seed, T=5, H=4, W=8, heads=2, d=8):
    rng = np.random.default_rng(seed)
    N = T * H * W
    q, k, v = (rng.standard_normal((1, N, heads, d)) for _ in range(3))
    return q, k, v, O.video_blocks(T, H, W)


def test_sparse_all_blocks_equals_dense():
    q, k, v, blocks = _sparse_case(2)
    nb = len(blocks)
    sel = [[[np.arange(nb) for _ in range(nb)] for _ in range(2)]]
    o = O.sparse_attn(q, k, v, blocks, sel, 0.3)
    od, _ = O.joint_attn(q, k, v, 0.3)
    assert np.allclose(o, od, atol=1e-12)


def test_sparse_single_block():
    q, k, v, blocks = _sparse_case(3)
    nb = len(blocks)
    sel = [[[np.array([(i + 1) % nb]) for i in range(nb)] for _ in range(2)]]
    o = O.sparse_attn(q, k, v, blocks, sel, 0.3)
    for i, (s, n) in enumerate(blocks):
        js, jn = blocks[(i + 1) % nb]
        for h in range(2):
            ref, _ = O.attn(q[0, s:s + n, h], k[0, js:js + jn, h], v[0, js:js + jn, h], 0.3)
            assert np.allclose(o[0, s:s + n, h], ref, atol=1e-13)


def test_sparse_order_of_selected_blocks_does_not_matter():
    q, k, v, blocks = _sparse_case(4)
    s0, n0 = blocks[1]
    a, la = O.sparse_attn_rows(q, k, v, blocks, [0, 2, 3], 0.3, 0, 1, 1)
    b, lb = O.sparse_attn_rows(q, k, v, blocks, [3, 0, 2], 0.3, 0, 1, 1)
    assert np.allclose(a, b, atol=1e-13) and np.allclose(la, lb, atol=1e-13)
