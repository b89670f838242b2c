"""Pins of the oracle's top-M truncation (O4'), the baseline that the
"Accurate Block Attention" abstract contrasts with its sampler: blocks scored
from the same estimates but kept by rank, with no reweighting.

The oracle sorts by (fixed-point estimate descending, index ascending).  The
checks below use other characterisations of the same set: the exchange
invariant, a repeated-maximum selection, and maximal total mass.
"""
import itertools

import numpy as np
import pytest

import oracle


def _fixed(p_row):
    # the fixed-point weights the sampler ranks on (O4's own conversion, pinned
    # by the sampler tests)
    P, _, _, _, _ = oracle.inclusion(p_row, 0)
    return P


def _rows(seed, nrows, nK, ties):
    rng = np.random.default_rng(seed)
    p = rng.dirichlet(np.full(nK, 0.3), size=nrows).astype(np.float32)
    if ties:
        # coarse values: many exact ties, and some zero rows / entries
        p = np.round(p * 8) / 8
        p[0] = 0
    return p


@pytest.mark.parametrize("nK,bp,ties", [(40, 1000, False), (40, 2500, True), (300, 800, True),
                                        (7, 5000, True), (64, 10000, False), (64, 0, True)])
def test_kept_set_dominates_the_dropped_one(nK, bp, ties):
    p = _rows(nK + bp, 25, nK, ties)
    counts, idx, logw, over = oracle.topk(p, bp)
    M = oracle.budget_blocks(bp, nK)
    assert not over
    for r in range(len(p)):
        kept = idx[r, :counts[r]]
        assert counts[r] == min(M, nK)
        assert np.all(np.diff(kept) > 0)
        assert np.all(logw[r, :counts[r]] == 0)
        P = _fixed(p[r])
        dropped = np.setdiff1d(np.arange(nK), kept)
        for a in kept:
            for b in dropped:
                assert P[a] > P[b] or (P[a] == P[b] and a < b), (r, a, b)


def test_repeated_maximum_selection():
    # pick the largest remaining (first index on ties) M times
    p = _rows(3, 40, 12, True)
    for bp in (900, 2600, 5000):
        counts, idx, _, _ = oracle.topk(p, bp)
        M = oracle.budget_blocks(bp, 12)
        for r in range(len(p)):
            P = _fixed(p[r]).astype(object)
            left = list(range(12))
            chosen = []
            for _ in range(min(M, 12)):
                best = max(left, key=lambda b: (P[b], -b))
                chosen.append(best)
                left.remove(best)
            assert sorted(chosen) == idx[r, :counts[r]].tolist()


def test_kept_set_has_the_largest_total_estimate():
    p = _rows(11, 30, 9, False)
    bp = 3400
    M = oracle.budget_blocks(bp, 9)
    counts, idx, _, _ = oracle.topk(p, bp)
    for r in range(len(p)):
        P = _fixed(p[r])
        best = max(sum(int(P[b]) for b in c) for c in itertools.combinations(range(9), M))
        assert sum(int(P[b]) for b in idx[r, :counts[r]]) == best


def test_keep_all_and_empty_budget():
    p = _rows(5, 4, 50, False)
    c, i, lw, _ = oracle.topk(p, 10000)
    assert np.all(c == 50) and np.all(i == np.arange(50))
    c, _, _, _ = oracle.topk(p, 0)
    assert np.all(c == 0)
    c, i, _, over = oracle.topk(p, 5000, capacity=10)
    assert over and np.all(c == 10)
