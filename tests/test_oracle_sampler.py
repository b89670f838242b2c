"""Pins for oracle O4 (SIP sampler).

- Budget rounding M = round-half-up(budget * nK) on worked values.
- The inclusion probabilities pi_b = min(1, c p_b) sum to M exactly
  (checked in exact rational arithmetic with Python fractions).
- c is checked against an independent exact solver (sort the fixed-point
  weights, try each saturation count, keep the consistent one) - a different
  algorithm from the oracle's water-filling.
- Empirical inclusion counts over 10^4 seeds are not in an exact binomial
  tail of probability 1e-7 around pi_b (so the Philox draw is compared in
  the right direction against the right threshold).
- log-weights equal the fp32 rounding of -ln(pi) computed with Python's
  float64 math.log, except where the oracle flags the rounding as too close
  to call.
- keep-all (M >= nK) and empty budgets; list order, determinism, capacity.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from block_sparse_attention_20_b200 import synth


@pytest.mark.parametrize("bp,nK,M", [(1000, 2048, 205), (800, 4725, 378), (1100, 7425, 817),
                                      (1000, 256, 26), (10000, 100, 100), (0, 50, 0),
                                      (50, 10, 0), (5000, 3, 2), (2500, 2, 1)])
def test_budget_rounding(bp, nK, M):
    assert oracle.budget_blocks(bp, nK) == M


def _exact_pi(P, M):
    """Independent exact solution of sum_b min(1, c P_b) = M (fractions)."""
    order = sorted(range(len(P)), key=lambda b: -P[b])
    total = sum(P)
    for k in range(0, M + 1):
        rest = total - sum(P[b] for b in order[:k])
        if rest == 0:
            break
        c = Fraction(M - k, rest)
        sat_ok = all(c * P[b] >= 1 for b in order[:k])
        unsat_ok = all(c * P[b] < 1 for b in order[k:])
        if sat_ok and unsat_ok:
            return [Fraction(1) if i in set(order[:k]) else c * P[i] for i in range(len(P))]
    # every positive block saturated, the rest have pi = 0
    return [Fraction(1) if P[b] > 0 else Fraction(0) for b in range(len(P))]


def _oracle_pi(P, sat, R, T):
    return [Fraction(1) if s else (Fraction(R * int(p), T) if T else Fraction(0))
            for p, s in zip(P, sat)]


@pytest.mark.parametrize("nK,M,conc,seed", [(16, 5, 0.3, 1), (16, 3, 0.1, 2), (12, 7, 1.0, 3),
                                             (64, 20, 0.05, 4), (200, 26, 0.3, 5),
                                             (16, 15, 0.2, 6)])
def test_inclusion_exact(nK, M, conc, seed):
    p = synth.random_probs(8, nK, seed, conc)
    for row in p:
        P, sat, R, T, rounds = oracle.inclusion(row, M)
        assert np.array_equal(P, [round(Fraction(float(x)) * 2**48) for x in row])
        pi = _oracle_pi([int(x) for x in P], sat, R, T)
        if sum(1 for x in P if x > 0) >= M:
            assert sum(pi) == M
        assert all(0 <= x <= 1 for x in pi)
        assert pi == _exact_pi([int(x) for x in P], M)


def test_inclusion_degenerate_rows():
    # all mass on 3 blocks, M = 5: those 3 saturate, nothing else can be drawn
    p = np.zeros(16, dtype=np.float32)
    p[[1, 7, 9]] = [0.5, 0.25, 0.25]
    P, sat, R, T, _ = oracle.inclusion(p, 5)
    assert list(np.nonzero(sat)[0]) == [1, 7, 9] and T == 0
    # uniform p: every pi = M / nK, no saturation
    p = np.full(40, 1.0 / 40, dtype=np.float32)
    P, sat, R, T, _ = oracle.inclusion(p, 10)
    assert not sat.any() and R == 10
    # NaN and negatives are read as 0, values above 1 as 1
    p = np.array([np.nan, -1.0, 2.0, 0.5], dtype=np.float32)
    P, sat, R, T, _ = oracle.inclusion(p, 1)
    assert list(P) == [0, 0, 2**48, 2**47]


def test_keep_all_and_empty():
    shape = (1, 1, 256, 8)
    p = synth.random_probs(2, 16, 7)
    counts, idx, logw, amb, of = oracle.sample(p, shape, [0, 1], 10000, 3)
    assert list(counts) == [16, 16]
    assert np.array_equal(idx, np.tile(np.arange(16), (2, 1)))
    assert np.all(logw == 0)
    counts, idx, logw, amb, of = oracle.sample(p, shape, [0, 1], 0, 3)
    assert list(counts) == [0, 0]


def test_inclusion_frequency_and_logw():
    nK, bp = 64, 2000  # M = 13
    shape = (1, 2, nK * 16, 8)
    p = synth.random_probs(1, nK, 11, 0.2)
    M = oracle.budget_blocks(bp, nK)
    P, sat, R, T, _ = oracle.inclusion(p[0], M)
    pi = np.array([float(x) for x in _oracle_pi([int(v) for v in P], sat, R, T)])
    nseed = 10000
    hits = np.zeros(nK)
    row = 3  # (beta=0, h=0, i=3) for nQ = 8
    for s in range(nseed):
        counts, idx, logw, amb, of = oracle.sample(p, shape, [row], bp, s)
        L = counts[0]
        sel = idx[0, :L]
        assert np.all(np.diff(sel) > 0)
        hits[sel] += 1
        for b, lw, a in zip(sel, logw[0, :L], amb[0, :L]):
            if sat[b]:
                assert lw == 0.0
            else:
                x = float(R * int(P[b])) / float(T)
                ref = np.float32(-math.log(x))
                assert a or lw == ref
    from scipy.stats import binom

    lo = binom.cdf(hits, nseed, pi)  # P(X <= hits)
    hi = binom.sf(hits - 1, nseed, pi)  # P(X >= hits)
    assert np.all(np.minimum(lo, hi) > 1e-7), (hits, pi * nseed)
    assert abs(hits.sum() / nseed - M) < 0.1


def test_rows_draw_independently_and_deterministically():
    nK = 32
    shape = (2, 3, nK * 16, 8)  # nQ = 4
    p = np.tile(synth.random_probs(1, nK, 13, 0.5), (24, 1))
    rows = np.arange(24)
    a = oracle.sample(p, shape, rows, 3000, 99)
    b = oracle.sample(p, shape, rows, 3000, 99)
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[0], b[0])
    sets = {tuple(a[1][r, :a[0][r]]) for r in rows}
    assert len(sets) > 12  # same p, different (beta, h, i) -> different draws
    c = oracle.sample(p, shape, rows, 3000, 100)
    assert not np.array_equal(a[1], c[1])


def test_capacity_truncates_and_flags():
    nK = 64
    shape = (1, 1, nK * 16, 8)
    p = synth.random_probs(1, nK, 17)
    full = oracle.sample(p, shape, [0], 5000, 1)
    L = int(full[0][0])
    cut = oracle.sample(p, shape, [0], 5000, 1, capacity=L - 3)
    assert cut[4] and cut[0][0] == L - 3
    assert np.array_equal(cut[1][0], full[1][0, :L - 3])
    ok = oracle.sample(p, shape, [0], 5000, 1, capacity=L)
    assert not ok[4]


# ---- paired draws (common random numbers across query blocks 2j, 2j+1) ----

def test_paired_rows_with_equal_probabilities_draw_equal_lists():
    # one uniform per (block, pair): equal p gives equal lists for the two rows
    # of a pair, while independent draws give different ones
    nK = 48
    shape = (2, 3, nK * 16, 8)  # nQ = 6: pairs (0,1), (2,3), (4,5) per head
    p = np.tile(synth.random_probs(1, nK, 21, 0.5), (36, 1))
    rows = np.arange(36)
    c, i, lw, _, _ = oracle.sample(p, shape, rows, 3000, 7, paired=True)
    for r in range(0, 36, 2):
        assert c[r] == c[r + 1] and np.array_equal(i[r, :c[r]], i[r + 1, :c[r]])
        assert np.array_equal(lw[r, :c[r]], lw[r + 1, :c[r]])
    ci, ii, _, _, _ = oracle.sample(p, shape, rows, 3000, 7)
    assert sum(ci[r] != ci[r + 1] or not np.array_equal(ii[r, :ci[r]], ii[r + 1, :ci[r]])
               for r in range(0, 36, 2)) >= 9
    # different pairs still draw differently
    assert len({tuple(i[r, :c[r]]) for r in range(0, 36, 2)}) > 12


def test_paired_draw_of_a_row_is_the_independent_draw_at_half_its_index():
    # under pairing, query blocks 2j and 2j+1 both draw with the counter that
    # query block j has without it
    nK = 40
    shape = (1, 2, nK * 16, 8)  # nQ = 5 (the last pair has one row)
    p = synth.random_probs(10, nK, 23, 0.3)
    rows = np.arange(10)
    cp, ip, lp, _, _ = oracle.sample(p, shape, rows, 2500, 11, paired=True)
    for r in rows:
        h, i = divmod(int(r), 5)
        half = h * 5 + (i >> 1)
        ce, ie, le, _, _ = oracle.sample(p[r:r + 1], shape, [half], 2500, 11)
        assert cp[r] == ce[0] and np.array_equal(ip[r, :cp[r]], ie[0, :ce[0]])
        assert np.array_equal(lp[r, :cp[r]], le[0, :ce[0]])


def test_paired_draws_take_a_block_in_both_rows_with_the_smaller_probability():
    # with one uniform U for both rows, block b is in both lists iff
    # U < min(pi_0b, pi_1b): P(both) = min(pi_0b, pi_1b), against pi_0b*pi_1b
    # for independent draws
    nK, bp = 32, 2500  # M = 8
    shape = (1, 1, nK * 16, 8)  # nQ = 2: one pair
    p = synth.random_probs(2, nK, 29, 0.4)
    M = oracle.budget_blocks(bp, nK)
    pis = []
    for r in range(2):
        P, sat, R, T, _ = oracle.inclusion(p[r], M)
        pis.append(np.array([float(x) for x in _oracle_pi([int(v) for v in P], sat, R, T)]))
    nseed = 4000
    both = np.zeros(nK)
    for s in range(nseed):
        c, i, _, _, _ = oracle.sample(p, shape, [0, 1], bp, s, paired=True)
        both[np.intersect1d(i[0, :c[0]], i[1, :c[1]])] += 1
    from scipy.stats import binom

    want = np.minimum(pis[0], pis[1])
    lo = binom.cdf(both, nseed, want)
    hi = binom.sf(both - 1, nseed, want)
    assert np.all(np.minimum(lo, hi) > 1e-7), (both, want * nseed)
    # and not the independent rate where the two differ noticeably
    gap = want - pis[0] * pis[1]
    assert np.all(both[gap > 0.1] / nseed > (pis[0] * pis[1])[gap > 0.1] + 0.05)


def test_slice_with_offsets_draws_what_the_whole_problem_draws():
    # the counter carries global (batch, head) indices: heads [1, 3) of batch 1
    # of a 2 x 3-head problem, drawn as a 1 x 2-head tensor with
    # batch_offset=1, head_offset=1, give the whole problem's lists
    B, H, N, Bk = 2, 3, 4000, 16
    nK, nQ = -(-N // Bk), -(-N // 128)
    rows = np.arange(B * H * nQ)
    p = synth.random_probs(len(rows), nK, 808, 0.2)
    whole = oracle.sample(p, (B, H, N, 64), rows, 900, 4242, Bk=Bk)
    sel = np.array([(1 * H + h) * nQ + i for h in (1, 2) for i in range(nQ)])
    part = oracle.sample(p[sel], (1, 2, N, 64), np.arange(2 * nQ), 900, 4242, Bk=Bk,
                         batch_offset=1, head_offset=1)
    assert np.array_equal(part[0], whole[0][sel])
    for k, r in enumerate(sel):
        L = whole[0][r]
        assert np.array_equal(part[1][k, :L], whole[1][r, :L])
        assert np.array_equal(part[2][k, :L], whole[2][r, :L])
    # without the offsets the slice draws other blocks
    plain = oracle.sample(p[sel], (1, 2, N, 64), np.arange(2 * nQ), 900, 4242, Bk=Bk)
    assert any(not np.array_equal(plain[1][k, :plain[0][k]], whole[1][r, :whole[0][r]])
               for k, r in enumerate(sel))
