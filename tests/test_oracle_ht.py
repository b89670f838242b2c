"""Pins for oracle O5 (attention on drawn blocks with log-weights).

- K1 keep-all: every block drawn with weight 1 reproduces dense attention
  (torch float64 softmax attention, a library routine) to 1e-12.
- K3 brute force: for nK = 16 all 2^16 draw outcomes are enumerated with
  their Poisson probabilities; the exact expectation of the weighted
  numerator and denominator equals the dense sums (1e-12 relative).  A wrong
  sign of the log-weight, a dropped block or a misplaced key index fails.
- K2 Monte Carlo: over 10^4 seeds of the real sampler, the mean weighted
  numerator/denominator match the dense sums within 4.5 standard errors of
  the closed-form Poisson-sampling variance sum_b (1-pi_b)/pi_b A_b^2.
- Uniform p: all pi are equal, the weights cancel in the ratio, and the
  output equals plain attention over the drawn keys (torch masked softmax).
- An empty list gives O = 0 and lse = -inf.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_20_b200 import synth


def _qkv(B, H, N, d, seed):
    return (synth.random_bf16((B, H, N, d), seed), synth.random_bf16((B, H, N, d), seed + 1),
            synth.random_bf16((B, H, N, d), seed + 2))


def _dense_sums(Q, K, V, h, i, Bq, Bk, N, d, nq):
    """Per query: dense row max m, and per-block A_b (den) and A_b (num)."""
    q = Q[0, h, i * Bq:i * Bq + nq].double()
    s = q @ K[0, h].double().T / math.sqrt(d)
    m = s.max(dim=1, keepdim=True).values
    e = torch.exp(s - m)
    nK = -(-N // Bk)
    blk = torch.arange(N) // Bk
    Aden = torch.zeros(nq, nK, dtype=torch.float64).index_add_(1, blk, e)
    Anum = torch.zeros(nq, nK, d, dtype=torch.float64)
    ev = e[:, :, None] * V[0, h].double()[None]
    Anum.index_add_(1, blk, ev)
    return Aden.numpy(), Anum.numpy()


@pytest.mark.parametrize("N,d,Bq,Bk", [(300, 32, 128, 16), (256, 64, 128, 32), (77, 8, 32, 4)])
def test_keep_all_equals_dense(N, d, Bq, Bk):
    Q, K, V = _qkv(1, 2, N, d, 31)
    nQ, nK = -(-N // Bq), -(-N // Bk)
    rows = np.arange(2 * nQ)
    counts = np.full(len(rows), nK, dtype=np.int32)
    idx = np.tile(np.arange(nK, dtype=np.int32), (len(rows), 1))
    logw = np.zeros((len(rows), nK))
    O, lse = oracle.ht_attention(Q, K, V, (1, 2, N, d), rows, counts, idx, logw, Bq=Bq, Bk=Bk)
    s = torch.einsum("bhnd,bhmd->bhnm", Q.double(), K.double()) / math.sqrt(d)
    ref = torch.einsum("bhnm,bhmd->bhnd", torch.softmax(s, -1), V.double()).numpy()
    ref_lse = torch.logsumexp(s, -1).numpy()
    for r in rows:
        h, i = divmod(int(r), nQ)
        n = min(Bq, N - i * Bq)
        assert np.allclose(O[r, :n], ref[0, h, i * Bq:i * Bq + n], rtol=0, atol=1e-12)
        assert np.allclose(lse[r, :n], ref_lse[0, h, i * Bq:i * Bq + n], rtol=0, atol=1e-12)


def test_brute_force_expectation_is_dense():
    N, d, Bq, Bk = 64, 8, 128, 4
    nK = 16
    Q, K, V = _qkv(1, 1, N, d, 41)
    p = synth.random_probs(1, nK, 42, 0.4)[0]
    P, sat, R, T, _ = oracle.inclusion(p, 6)
    pi = np.array([1.0 if s else R * int(x) / T for x, s in zip(P, sat)])
    assert np.all(pi > 0)
    nq = 3
    subsets = list(itertools.product([0, 1], repeat=nK))
    S = np.array(subsets, dtype=bool)
    # outcomes that drop a saturated block have probability 0; keep the rest
    S = S[np.all(S[:, sat] | ~sat[None, :], axis=1)]
    prob = np.prod(np.where(S, pi[None], 1.0 - pi[None]), axis=1)
    assert abs(prob.sum() - 1.0) < 1e-12
    counts = S.sum(1).astype(np.int32)
    idx = np.full((len(S), nK), 0, dtype=np.int32)
    logw = np.zeros((len(S), nK))
    lwb = -np.log(pi)
    for k, row in enumerate(S):
        sel = np.nonzero(row)[0]
        idx[k, :len(sel)] = sel
        logw[k, :len(sel)] = lwb[sel]
    rows = np.zeros(len(S), dtype=np.int64)
    O, lse, num, den = oracle.ht_attention(Q, K, V, (1, 1, N, d), rows, counts, idx, logw,
                                           Bq=Bq, Bk=Bk, nq_max=nq, want_numden=True)
    Aden, Anum = _dense_sums(Q, K, V, 0, 0, Bq, Bk, N, d, nq)
    Eden = (prob[:, None] * den[:, :nq]).sum(0)
    Enum = (prob[:, None, None] * num[:, :nq]).sum(0)
    assert np.allclose(Eden, Aden.sum(1), rtol=1e-12, atol=0)
    assert np.allclose(Enum, Anum.sum(1), rtol=1e-12, atol=1e-12)


def test_monte_carlo_unbiased():
    N, d, Bq, Bk = 512, 16, 128, 16
    nK, bp = 32, 2500
    Q, K, V = _qkv(1, 1, N, d, 51)
    shape = (1, 1, N, d)
    row = 1
    _, p32 = oracle.block_probs(Q, K, shape, [row], 2, 3, Bq=Bq, Bk=Bk)
    P, sat, R, T, _ = oracle.inclusion(p32[0], oracle.budget_blocks(bp, nK))
    pi = np.array([1.0 if s else R * int(x) / T for x, s in zip(P, sat)])
    nq, nseed = 4, 10000
    sum_den = np.zeros(nq)
    sum_num = np.zeros((nq, d))
    for s in range(nseed):
        counts, idx, logw, amb, of = oracle.sample(p32, shape, [row], bp, s, Bq=Bq, Bk=Bk)
        O, lse, num, den = oracle.ht_attention(Q, K, V, shape, [row], counts, idx, logw,
                                               Bq=Bq, Bk=Bk, nq_max=nq, want_numden=True,
                                               nthreads=1)
        sum_den += den[0, :nq]
        sum_num += num[0, :nq]
    Aden, Anum = _dense_sums(Q, K, V, 0, row, Bq, Bk, N, d, nq)
    live = pi > 0
    w = np.where(live, (1 - pi) / np.where(live, pi, 1.0), 0.0)
    # blocks with pi = 0 are never drawn: the estimator's mean excludes them
    ref_den = (Aden * live).sum(1)
    ref_num = (Anum * live[None, :, None]).sum(1)
    se_den = np.sqrt((w[None] * Aden**2).sum(1) / nseed)
    se_num = np.sqrt((w[None, :, None] * Anum**2).sum(1) / nseed)
    assert np.all(np.abs(sum_den / nseed - ref_den) <= 4.5 * se_den + 1e-12)
    assert np.all(np.abs(sum_num / nseed - ref_num) <= 4.5 * se_num + 1e-12)
    # the excluded mass (p below 2^-48 resolution) is negligible here
    assert np.all((Aden * ~live).sum(1) <= 1e-9 * Aden.sum(1))


def test_uniform_p_equals_masked_attention():
    N, d, Bq, Bk = 384, 16, 128, 16
    nK = 24
    Q, K, V = _qkv(1, 1, N, d, 61)
    shape = (1, 1, N, d)
    p = np.full((3, nK), 1.0 / nK, dtype=np.float32)
    rows = np.arange(3)
    counts, idx, logw, amb, of = oracle.sample(p, shape, rows, 3000, 5, Bq=Bq, Bk=Bk)
    assert len(set(logw[counts > 0][:, 0])) == 1
    O, lse = oracle.ht_attention(Q, K, V, shape, rows, counts, idx, logw, Bq=Bq, Bk=Bk)
    for r in rows:
        mask = torch.zeros(N, dtype=torch.bool)
        for b in idx[r, :counts[r]]:
            mask[b * Bk:(b + 1) * Bk] = True
        q = Q[0, 0, r * Bq:(r + 1) * Bq].double()
        s = (q @ K[0, 0].double().T / math.sqrt(d)).masked_fill(~mask, -math.inf)
        ref = torch.softmax(s, -1) @ V[0, 0].double()
        assert np.allclose(O[r], ref.numpy(), rtol=0, atol=1e-12)


def test_empty_list():
    N, d = 256, 8
    Q, K, V = _qkv(1, 1, N, d, 71)
    O, lse = oracle.ht_attention(Q, K, V, (1, 1, N, d), [0], [0], np.zeros((1, 16), np.int32),
                                 np.zeros((1, 16)), Bk=16)
    assert np.all(O == 0) and np.all(np.isneginf(lse))
