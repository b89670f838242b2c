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


# --------------------------------------------------------------- coarse scoring

def _symmetric_blocks(seed, B, H, N, d, Bk):
    """K whose every block mean is exactly a bf16 vector: each block holds a
    centre c_b (bf16) and pairs c_b + e, c_b - e (exact in bf16), so the mean of
    its keys is c_b; a ragged last block holds only centres.  Returns K and the
    keys replaced by their block means (same shape)."""
    import torch
    rng = np.random.default_rng(seed)
    nK = -(-N // Bk)
    K = np.zeros((B, H, N, d), np.float32)
    Kbar = np.zeros_like(K)
    for b in range(nK):
        lo, hi = b * Bk, min(N, (b + 1) * Bk)
        n = hi - lo
        c = rng.integers(-8, 9, size=(B, H, 1, d)).astype(np.float32) / 8  # exact in bf16
        K[:, :, lo:hi] = c
        Kbar[:, :, lo:hi] = c
        for u in range(0, n - 1 if n % 2 else n, 2):
            e = rng.integers(-4, 5, size=(B, H, d)).astype(np.float32) / 16
            K[:, :, lo + u] = c[:, :, 0] + e
            K[:, :, lo + u + 1] = c[:, :, 0] - e
    to = lambda x: torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(to(K).float().numpy(), K)  # every value exact in bf16
    return to(K), to(Kbar)


def test_coarse_equals_per_key_rule_on_block_mean_keys():
    B, H, N, d, Bk = 1, 2, 300, 64, 16  # 19 blocks, the last with 12 keys
    import torch
    rng = np.random.default_rng(4)
    Q = torch.from_numpy(rng.standard_normal((B, H, N, d)).astype(np.float32)).to(torch.bfloat16)
    K, Kbar = _symmetric_blocks(9, B, H, N, d, Bk)
    rows = np.arange(B * H * 3)
    pc, _ = oracle.block_probs(Q, K, (B, H, N, d), rows, 4, 3, Bk=Bk, coarse=True)
    pk, _ = oracle.block_probs(Q, Kbar, (B, H, N, d), rows, 4, 3, Bk=Bk, coarse=False)
    assert np.allclose(pc, pk, rtol=0, atol=1e-12)
    assert np.allclose(pc.sum(1), 1.0, atol=1e-12)
    # and the coarse rule really differs from the per-key one on K itself
    pf, _ = oracle.block_probs(Q, K, (B, H, N, d), rows, 4, 3, Bk=Bk, coarse=False)
    assert np.max(np.abs(pf - pc)) > 1e-6


def test_coarse_equals_per_key_when_blocks_hold_one_key_value():
    B, H, N, d, Bk = 1, 1, 200, 64, 32
    import torch
    rng = np.random.default_rng(8)
    Q = torch.from_numpy(rng.standard_normal((B, H, N, d)).astype(np.float32)).to(torch.bfloat16)
    k = rng.standard_normal((B, H, -(-N // Bk), d)).astype(np.float32)
    K = torch.from_numpy(np.repeat(k, Bk, axis=2)[:, :, :N]).to(torch.bfloat16)
    rows = np.arange(2)
    pc, _ = oracle.block_probs(Q, K, (B, H, N, d), rows, 2, 2, Bk=Bk, coarse=True)
    pk, _ = oracle.block_probs(Q, K, (B, H, N, d), rows, 2, 2, Bk=Bk, coarse=False)
    assert np.allclose(pc, pk, rtol=0, atol=1e-12)
