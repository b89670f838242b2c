"""Pins for oracle O1 (dense attention) and O2 (per-query-block k-means).

O1 is checked against torch's float64 CPU softmax attention (a library
routine, not the oracle's loops).  O2 is checked against scikit-learn's Lloyd
k-means started from the same seeds, against its defining invariants
(centroid = mean of members, sizes = member counts, distortion never rises)
and against the special cases C=1 (block mean) and C=n (every row its own
cluster, zero distortion).
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_20_b200 import synth


def _qkv(B, H, N, d, seed):
    return (synth.random_bf16((B, H, N, d), seed), synth.random_bf16((B, H, N, d), seed + 1),
            synth.random_bf16((B, H, N, d), seed + 2))


def _torch_dense(Q, K, V, scale):
    q, k, v = Q.double(), K.double(), V.double()
    s = torch.einsum("bhnd,bhmd->bhnm", q, k) * scale
    return torch.einsum("bhnm,bhmd->bhnd", torch.softmax(s, dim=-1), v)


@pytest.mark.parametrize("N,d,Bq", [(300, 32, 128), (64, 8, 16), (129, 16, 128)])
def test_dense_matches_torch_f64(N, d, Bq):
    B, H = 2, 2
    Q, K, V = _qkv(B, H, N, d, 11)
    nQ = -(-N // Bq)
    rows = np.arange(B * H * nQ)
    O, lse = oracle.dense_attention(Q, K, V, (B, H, N, d), rows, Bq=Bq, want_lse=True)
    ref = _torch_dense(Q, K, V, 1.0 / np.sqrt(d)).numpy()
    s = torch.einsum("bhnd,bhmd->bhnm", Q.double(), K.double()) / np.sqrt(d)
    ref_lse = torch.logsumexp(s, dim=-1).numpy()
    for r in rows:
        bh, i = divmod(int(r), nQ)
        b, h = divmod(bh, H)
        n = min(Bq, N - i * Bq)
        got = O[r, :n]
        exp = ref[b, h, i * Bq:i * Bq + n]
        assert np.max(np.abs(got - exp)) <= 1e-12 * max(1.0, np.max(np.abs(exp)))
        assert np.all(O[r, n:] == 0)
        assert np.allclose(lse[r, :n], ref_lse[b, h, i * Bq:i * Bq + n], rtol=0, atol=1e-12)


def _block_rows(Q, b, h, i, Bq, N):
    n = min(Bq, N - i * Bq)
    return Q[b, h, i * Bq:i * Bq + n].double().numpy()


def test_kmeans_matches_sklearn_lloyd():
    """Round by round: oracle state after k rounds vs one sklearn Lloyd round
    started from the oracle's state after k-1 rounds.  Rounds in which a
    cluster is empty are skipped (sklearn relocates empty clusters)."""
    from sklearn.cluster import KMeans

    w = synth.TINY
    Q, K, V = synth.generate(w, heads=1)
    shape = (1, 1, w.N, w.d)
    rows = np.arange(w.nQ)
    C, I = 4, 5
    prev = None
    checked = 0
    for k in range(1, I + 1):
        cent, cnt, asg = oracle.kmeans(Q, shape, rows, C, k)
        for i in rows:
            X = _block_rows(Q, 0, 0, i, 128, w.N)
            n = len(X)
            init = X[[j * n // C for j in range(C)]] if k == 1 else prev[i]
            if len(np.unique(init, axis=0)) < C or np.min(cnt[i]) == 0:
                continue
            km = KMeans(n_clusters=C, init=init, n_init=1, max_iter=1, tol=0.0,
                        algorithm="lloyd").fit(X)
            assert np.allclose(cent[i], km.cluster_centers_, rtol=0, atol=1e-9), (k, i)
            checked += 1
        prev = cent
    assert checked >= I * w.nQ // 2


@pytest.mark.parametrize("N,Bq,C", [(4096, 128, 4), (300, 128, 8), (100, 32, 5)])
def test_kmeans_invariants(N, Bq, C):
    d = 16
    Q = synth.random_bf16((1, 2, N, d), 5)
    nQ = -(-N // Bq)
    rows = np.arange(2 * nQ)
    I = 6
    cent, cnt, asg, trace = oracle.kmeans(Q, (1, 2, N, d), rows, C, I, Bq=Bq, want_trace=True)
    for r in rows:
        h, i = divmod(int(r), nQ)
        X = _block_rows(Q, 0, h, i, Bq, N)
        n = len(X)
        a = asg[r, :n]
        assert np.all(asg[r, n:] == -1)
        ce = min(C, n)
        assert a.min() >= 0 and a.max() < ce
        assert np.array_equal(np.bincount(a, minlength=C), cnt[r])
        for j in range(ce):
            if cnt[r, j]:
                assert np.allclose(cent[r, j], X[a == j].mean(axis=0), rtol=0, atol=1e-12)
        t = trace[r]
        assert np.all(np.diff(t) <= 1e-9 * max(1.0, t[0])), t


def test_kmeans_special_cases():
    N, d, Bq = 200, 12, 64
    Q = synth.random_bf16((1, 1, N, d), 9)
    nQ = -(-N // Bq)
    rows = np.arange(nQ)
    cent, cnt, asg = oracle.kmeans(Q, (1, 1, N, d), rows, 1, 3, Bq=Bq)
    for i in rows:
        X = _block_rows(Q, 0, 0, i, Bq, N)
        assert np.allclose(cent[i, 0], X.mean(axis=0), rtol=0, atol=1e-12)
        assert cnt[i, 0] == len(X)
    # C = Bq: every row is its own centroid, zero distortion (rows distinct).
    cent, cnt, asg, tr = oracle.kmeans(Q, (1, 1, N, d), rows, Bq, 2, Bq=Bq, want_trace=True)
    for i in rows:
        X = _block_rows(Q, 0, 0, i, Bq, N)
        n = len(X)
        assert np.array_equal(asg[i, :n], np.arange(n))
        assert np.allclose(cent[i, :n], X, rtol=0, atol=0)
        assert np.all(cnt[i, :n] == 1) and np.all(cnt[i, n:] == 0)
        assert tr[i, -1] == 0.0
