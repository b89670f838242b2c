"""Pins for oracle O3 (IBCS block probabilities).

- Each row of p is a probability vector over key blocks (sums to 1, >= 0).
- C = n (every query its own centroid): p equals the mean, over the block's
  queries, of their dense attention mass per key block, computed here with
  torch's float64 softmax (library routine).  This catches a wrong scale,
  sign, index or transposed operand anywhere in the scoring.
- C = 1: the single centroid is the mean query, so p is the softmax mass of
  the mean query per key block (torch float64 softmax).
- Ragged tails in both the query and the key dimension.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_20_b200 import synth


def _mass_ref(qrows, K, N, Bk, scale):
    """Mean over qrows of softmax(scale * q.K) summed per key block."""
    s = torch.from_numpy(qrows) @ K.T * scale
    pr = torch.softmax(s, dim=-1).mean(0).numpy()
    nK = -(-N // Bk)
    pad = np.zeros(nK * Bk)
    pad[:N] = pr
    return pad.reshape(nK, Bk).sum(1)


@pytest.mark.parametrize("N,d,Bq,Bk", [(296, 16, 32, 8), (200, 8, 64, 16)])
def test_block_probs_special_cases(N, d, Bq, Bk):
    Q = synth.random_bf16((1, 2, N, d), 21)
    K = synth.random_bf16((1, 2, N, d), 22)
    nQ = -(-N // Bq)
    rows = np.arange(2 * nQ)
    scale = 1.0 / np.sqrt(d)
    for C in (Bq, 1):
        p64, p32 = oracle.block_probs(Q, K, (1, 2, N, d), rows, C, 3, Bq=Bq, Bk=Bk)
        assert np.allclose(p64.sum(1), 1.0, rtol=0, atol=1e-12)
        assert np.all(p64 >= 0)
        assert np.array_equal(p32, p64.astype(np.float32))
        for r in rows:
            h, i = divmod(int(r), nQ)
            X = Q[0, h, i * Bq:min(N, (i + 1) * Bq)].double().numpy()
            Kh = K[0, h].double()
            if C == 1:
                ref = _mass_ref(X.mean(0, keepdims=True), Kh, N, Bk, scale)
            else:
                ref = _mass_ref(X, Kh, N, Bk, scale)
            assert np.allclose(p64[r], ref, rtol=0, atol=1e-12), (C, r)


def test_block_probs_sum_to_one_on_video_tokens():
    w = synth.TINY
    Q, K, V = synth.generate(w, heads=2)
    rows = np.arange(2 * w.nQ)
    p64, p32 = oracle.block_probs(Q, K, (1, 2, w.N, w.d), rows, w.clusters, w.iters,
                                  Bk=w.Bk)
    assert np.allclose(p64.sum(1), 1.0, rtol=0, atol=1e-12)
    assert np.all(np.abs(p32.astype(np.float64).sum(1) - 1.0) <= w.nK * 2.0**-24)
    # The prototype structure concentrates mass: the top 10% of blocks hold most of it.
    top = np.sort(p64, axis=1)[:, ::-1][:, : w.nK // 10].sum(1)
    assert np.median(top) > 0.5
