"""CPU tests of the parity bar for block selection (tests/_util.py
``selection_verdict``): a GPU set may differ from the oracle's only where fp32
rounding can move the cutoff of S_i = Top-k(P_i, k) U Top-p(P_i, p) (Prism
guide, Method section 3) -- a block tied in probability with the cutoff
block, or a top-p crossing one block earlier or later when the cumulative sum
that decides it is within the tolerance of p.  Everything else is rejected,
including an arbitrary set on a row whose top-p sum is near-tied."""
import numpy as np

import oracle as O

from _util import fp32_tie_tol, selection_matches, selection_verdict


def _probs(n, seed):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal(n) * 2.0
    e = np.exp(s - s.max())
    return e / e.sum()


def _ranked(P):
    return sorted(range(len(P)), key=lambda j: (-P[j], j))


def test_exact_and_plain_mismatches():
    P = _probs(40, 1)
    order = _ranked(P)
    ref = O.select_from_probs(P, 5, 0.6)
    assert selection_verdict(ref, ref, P, 5, 0.6) == "exact"
    m = len(ref)
    # the last selected block swapped for a block far below the cutoff
    bad = sorted(set(ref.tolist()) - {order[m - 1]} | {order[-1]})
    assert selection_verdict(np.array(bad), ref, P, 5, 0.6) == "mismatch"
    # one block short, one block too many (no tie anywhere)
    assert selection_verdict(ref[:-1], ref, P, 5, 0.6) == "mismatch"
    assert selection_verdict(np.array(sorted(order[:m + 1])), ref, P, 5, 0.6) == "mismatch"
    # duplicates and out-of-range ids
    assert selection_verdict(np.concatenate([ref[:-1], ref[:1]]), ref, P, 5, 0.6) == "mismatch"
    assert selection_verdict(np.concatenate([ref[:-1], [40]]), ref, P, 5, 0.6) == "mismatch"
    # a set far from the oracle's on a row without ties
    assert not selection_matches(np.array(sorted(order[-m:])), ref, P, 5, 0.6)


def test_value_tie_at_the_cutoff_allows_a_swap_only_between_tied_blocks():
    P = _probs(30, 2)
    order = _ranked(P)
    k = 6
    # make the 6th and 7th ranked blocks equal (within fp32 resolution)
    a, b = order[k - 1], order[k]
    P = P.copy()
    P[b] = P[a] * (1 - 3e-7)
    P /= P.sum()
    ref = O.select_from_probs(P, k, 0.0)  # top-p of 0 selects one block: top-k decides
    assert len(ref) == k and a in ref
    swapped = np.array(sorted(set(ref.tolist()) - {a} | {b}))
    assert selection_verdict(swapped, ref, P, k, 0.0) == "tie"
    # swapping the tied block for a clearly lower one is not a tie
    c = order[k + 3]
    wrong = np.array(sorted(set(ref.tolist()) - {a} | {c}))
    assert selection_verdict(wrong, ref, P, k, 0.0) == "mismatch"
    # dropping a top-ranked block to keep both tied ones is not a tie either
    wrong2 = np.array(sorted(set(ref.tolist()) - {order[0]} | {b}))
    assert selection_verdict(wrong2, ref, P, k, 0.0) == "mismatch"


def test_mass_tie_moves_the_top_p_cutoff_by_one_block_only():
    # P such that the cumulative sum of the first 5 ranked blocks is exactly p
    P = np.array([0.3, 0.2, 0.15, 0.1, 0.05, 0.04, 0.04, 0.03] + [0.01] * 9)
    P = P / P.sum()
    order = _ranked(P)
    p = float(np.cumsum(P[order])[4])  # crossing at block 5 (inclusive)
    ref = O.select_from_probs(P, 1, p)
    assert len(ref) in (5, 6)
    n5 = np.array(sorted(order[:5]))
    n6 = np.array(sorted(order[:6]))
    n4 = np.array(sorted(order[:4]))
    n7 = np.array(sorted(order[:7]))
    # the crossing sum equals p: one block more or one less are both fp32 outcomes
    assert selection_verdict(n5, ref, P, 1, p) != "mismatch"
    assert selection_verdict(n6, ref, P, 1, p) != "mismatch"
    assert selection_verdict(n4, ref, P, 1, p) == "mismatch"
    # 7 blocks is two past the crossing unless blocks 6 and 7 tie (they do here:
    # 0.04 and 0.04), in which case a 6-block set may hold either of them
    alt6 = np.array(sorted(order[:5] + [order[6]]))
    assert selection_verdict(alt6, ref, P, 1, p) == "tie"
    assert selection_verdict(n7, ref, P, 1, p) == "mismatch"


def test_garbage_on_a_near_tied_row_is_rejected():
    # A row whose top-p sum is within the tolerance of p: the old check
    # excused such rows entirely; now the set itself must still be right.
    P = np.array([0.25, 0.25, 0.2, 0.1, 0.1, 0.05, 0.05])
    order = _ranked(P)
    p = float(np.cumsum(P[order])[2])  # exactly 0.7
    ref = O.select_from_probs(P, 1, p)
    garbage = np.array(sorted(order[-len(ref):]))  # the same size, the lowest blocks
    assert selection_verdict(garbage, ref, P, 1, p) == "mismatch"
    missing_top = np.array(sorted(order[1:len(ref) + 1]))
    assert selection_verdict(missing_top, ref, P, 1, p) == "mismatch"


def test_fp32_tie_band_from_the_score_error_bound():
    # a row of near-uniform probabilities (a background query block): blocks
    # whose log-probabilities differ by less than the fp32 error bound of the
    # scores are ties; a wider gap is not
    rng = np.random.default_rng(4)
    d, n = 128, 50
    qbar = rng.standard_normal(d) * 0.05
    kbar = rng.standard_normal((n, d)) * 0.05
    scale = 1 / np.sqrt(d)
    ltol = fp32_tie_tol(qbar, kbar, scale, 64)
    assert np.all(ltol > 0) and np.all(ltol < 1e-5)
    # the bound: at least the d-term dot product's worst case
    a = np.abs(kbar * qbar).sum(1) * scale
    assert np.all(ltol >= 2.0 ** -24 * d * a)
    s = (kbar @ qbar) * scale
    P = np.exp(s - s.max())
    P /= P.sum()
    order = _ranked(P)
    k = 10
    a_, b_ = order[k - 1], order[k]
    # place block b_ just below a_, within and then beyond the tie band
    for factor, expect in ((0.5, "tie"), (3.0, "mismatch")):
        Q = P.copy()
        gap = factor * (ltol[a_] + ltol[b_])
        Q[b_] = Q[a_] * np.exp(-gap)
        ref = O.select_from_probs(Q, k, 0.0)
        swapped = np.array(sorted(set(ref.tolist()) - {a_} | {b_}))
        assert selection_verdict(swapped, ref, Q, k, 0.0, ltol=ltol) == expect
    # far below the cutoff is never a tie
    ref = O.select_from_probs(P, k, 0.0)
    wrong = np.array(sorted(set(ref.tolist()) - {order[k - 1]} | {order[-1]}))
    assert selection_verdict(wrong, ref, P, k, 0.0, ltol=ltol) == "mismatch"
