"""Float64 CPU oracle for the AB-Attention hot path (TEST INFRASTRUCTURE ONLY).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package.  It wraps ``oracle.c`` (plain C, float64) with ctypes and
numpy; it shares no code with the CUDA library and never imports it.

Parity status of each function, with the check that pins it, is listed in the
module docstrings of ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liborc.so")
_lock = threading.Lock()
_lib = None

# gcc flags: IEEE semantics (no fast-math, no FMA contraction) so the float64
# arithmetic is exactly what the C source says.
CFLAGS = ["-O2", "-std=gnu11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liborc.so next to it (idempotent)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, u64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double
        lib.orc_philox4x32_10.argtypes = [P, P, P]
        lib.orc_philox4x32_10.restype = None
        lib.orc_dense_attention.argtypes = [P, P, P, i32, i32, i32, i32, i32, f64, P, i64, i32, P, P]
        lib.orc_kmeans.argtypes = [P, i32, i32, i32, i32, i32, i32, i32, P, i64, i32, P, P, P, P]
        lib.orc_block_probs.argtypes = [P, P, i32, i32, i32, i32, i32, i32, i32, i32, f64, i32,
                                        P, i64, i32, P, P]
        lib.orc_budget_blocks.argtypes = [i32, i32]
        lib.orc_budget_blocks.restype = i64
        lib.orc_inclusion.argtypes = [P, i32, i64, P, P, P, P, P]
        lib.orc_topk.argtypes = [P, i64, i32, i32, i32, i32, P, P, P]
        lib.orc_sample.argtypes = [P, i32, i32, i32, i32, i32, P, i64, i32, u64, i32, i32,
                                   P, P, P, P, i32, i32, i32]
        lib.orc_ht_attention.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, f64, P, i64,
                                         P, P, P, i32, i32, i32, P, P, P, P]
        lib.orc_forward.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, i32, i32, f64,
                                    u64, P, i64, i32, P, P, P, P, P, i32, i32]
        _lib = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bits(x) -> np.ndarray:
    """bf16 input as a C-contiguous uint16 array of bit patterns.

    Accepts a torch bfloat16 tensor (CPU) or a numpy uint16 array."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy inputs must be uint16 bf16 bit patterns")
        return np.ascontiguousarray(x)
    import torch
    if x.dtype != torch.bfloat16:
        raise TypeError("torch inputs must be bfloat16")
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _rows(rows) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _check(rc, what):
    if rc < 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")
    return rc


def philox4x32_10(ctr, key) -> np.ndarray:
    """Philox4x32-10 block: 4 counter words, 2 key words -> 4 output words."""
    lib = _load()
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32).reshape(4))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32).reshape(2))
    out = np.zeros(4, dtype=np.uint32)
    lib.orc_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def dense_attention(Q, K, V, shape, rows, Bq=128, scale=None, nthreads=None, want_lse=False):
    """O1: dense softmax attention for the listed query blocks.

    Returns O [nrows, Bq, d] float64 (rows past N are 0) and optionally lse."""
    B, H, N, d = shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    r = _rows(rows)
    O = np.zeros((len(r), Bq, d), dtype=np.float64)
    lse = np.zeros((len(r), Bq), dtype=np.float64) if want_lse else None
    q, k, v = _bits(Q), _bits(K), _bits(V)
    _check(_load().orc_dense_attention(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, Bq, scale,
                                       _ptr(r), len(r), nthreads or default_threads(),
                                       _ptr(O), _ptr(lse)), "dense_attention")
    return (O, lse) if want_lse else O


def kmeans(Q, shape, rows, C, iters, Bq=128, nthreads=None, want_trace=False):
    """O2: per-query-block Lloyd k-means.

    Returns centroids [nrows, C, d], counts [nrows, C], assign [nrows, Bq]
    (-1 for rows past N) and optionally the distortion trace [nrows, 2*iters]."""
    B, H, N, d = shape
    r = _rows(rows)
    cent = np.zeros((len(r), C, d), dtype=np.float64)
    cnt = np.zeros((len(r), C), dtype=np.int32)
    asg = np.zeros((len(r), Bq), dtype=np.int32)
    trace = np.zeros((len(r), 2 * iters), dtype=np.float64) if want_trace else None
    _check(_load().orc_kmeans(_ptr(_bits(Q)), B, H, N, d, Bq, C, iters, _ptr(r), len(r),
                              nthreads or default_threads(), _ptr(cent), _ptr(cnt), _ptr(asg),
                              _ptr(trace)), "kmeans")
    return (cent, cnt, asg, trace) if want_trace else (cent, cnt, asg)


def block_probs(Q, K, shape, rows, C, iters, Bq=128, Bk=16, scale=None, nthreads=None,
                coarse=False):
    """O3: IBCS block probabilities. Returns (p float64, p fp32) [nrows, nK].

    coarse=True: O3', each key block scored once through its mean key, its
    share n_b * exp(scale * c.kbar_b) normalised over the blocks."""
    B, H, N, d = shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    nK = -(-N // Bk)
    r = _rows(rows)
    p64 = np.zeros((len(r), nK), dtype=np.float64)
    p32 = np.zeros((len(r), nK), dtype=np.float32)
    _check(_load().orc_block_probs(_ptr(_bits(Q)), _ptr(_bits(K)), B, H, N, d, Bq, Bk, C, iters,
                                   scale, int(bool(coarse)), _ptr(r), len(r), nthreads or default_threads(),
                                   _ptr(p64), _ptr(p32)), "block_probs")
    return p64, p32


def budget_blocks(budget_bp: int, nK: int) -> int:
    """M, the expected number of drawn blocks per query block."""
    return int(_load().orc_budget_blocks(int(budget_bp), int(nK)))


def inclusion(p_row, M):
    """O4 water-filling for one row of fp32 probabilities.

    Returns (P int64 fixed-point, saturated bool, R, T, rounds)."""
    p = np.ascontiguousarray(np.asarray(p_row, dtype=np.float32).reshape(-1))
    nK = len(p)
    P = np.zeros(nK, dtype=np.int64)
    sat = np.zeros(nK, dtype=np.uint8)
    R = ctypes.c_int64()
    T = ctypes.c_int64()
    rounds = ctypes.c_int32()
    _check(_load().orc_inclusion(_ptr(p), nK, int(M), _ptr(P), _ptr(sat), ctypes.byref(R),
                                 ctypes.byref(T), ctypes.byref(rounds)), "inclusion")
    return P, sat.astype(bool), R.value, T.value, rounds.value


def sample(p, shape, rows, budget_bp, seed, Bq=128, Bk=16, capacity=None, nthreads=None,
           paired=False, batch_offset=0, head_offset=0):
    """O4: SIP draw for the listed rows (p is fp32 [nrows, nK]).

    paired=True: common random numbers -- query blocks 2j and 2j+1 of a head
    draw with the same Philox counter (floor(i/2) in place of i).
    batch_offset, head_offset: global index of the shape's first batch element
    and head when it is a slice of a larger problem (the counter's words 3, 2).

    Returns counts [nrows], idx [nrows, cap], logw fp32 [nrows, cap],
    amb uint8 [nrows, cap] (1 where the fp32 rounding of -ln(pi) is too close
    to call), overflow flag."""
    B, H, N, d = shape
    nK = -(-N // Bk)
    r = _rows(rows)
    p = np.ascontiguousarray(np.asarray(p, dtype=np.float32).reshape(len(r), nK))
    cap = nK if capacity is None else int(capacity)
    counts = np.zeros(len(r), dtype=np.int32)
    idx = np.full((len(r), cap), -1, dtype=np.int32)
    logw = np.zeros((len(r), cap), dtype=np.float32)
    amb = np.zeros((len(r), cap), dtype=np.uint8)
    rc = _check(_load().orc_sample(_ptr(p), B, H, N, Bq, Bk, _ptr(r), len(r), int(budget_bp),
                                   int(seed) & (2**64 - 1), cap, nthreads or default_threads(),
                                   _ptr(counts), _ptr(idx), _ptr(logw), _ptr(amb), int(bool(paired)),
                                   int(batch_offset), int(head_offset)),
                "sample")
    return counts, idx, logw, amb, bool(rc == 1)


def topk(p, budget_bp, capacity=None, nthreads=None):
    """O4': top-M truncation of fp32 probability rows p [nrows, nK]: the M
    largest (48-bit fixed point, ties to the lower index), ascending, log-weight
    0.  Returns counts [nrows], idx [nrows, cap], logw fp32 [nrows, cap],
    overflow flag."""
    p = np.ascontiguousarray(np.asarray(p, dtype=np.float32))
    nrows, nK = p.shape
    cap = nK if capacity is None else int(capacity)
    counts = np.zeros(nrows, dtype=np.int32)
    idx = np.full((nrows, cap), -1, dtype=np.int32)
    logw = np.zeros((nrows, cap), dtype=np.float32)
    rc = _load().orc_topk(_ptr(p), nrows, nK, int(budget_bp), cap, nthreads or default_threads(),
                          _ptr(counts), _ptr(idx), _ptr(logw))
    if rc < 0:
        raise RuntimeError(f"orc_topk failed ({rc})")
    return counts, idx, logw, bool(rc == 1)


def ht_attention(Q, K, V, shape, rows, counts, idx, logw, Bq=128, Bk=16, scale=None,
                 nq_max=None, want_numden=False, nthreads=None):
    """O5: attention on the drawn blocks with per-block log-weights.

    logw may be fp32 (widened exactly) or float64.  Returns O [nrows, Bq, d],
    lse [nrows, Bq] and, if asked, the HT numerator/denominator relative to
    the dense row maximum."""
    B, H, N, d = shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    r = _rows(rows)
    counts = np.ascontiguousarray(np.asarray(counts, dtype=np.int32).reshape(len(r)))
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(len(r), -1))
    cap = idx.shape[1]
    lw = np.ascontiguousarray(np.asarray(logw).astype(np.float64).reshape(len(r), cap))
    O = np.zeros((len(r), Bq, d), dtype=np.float64)
    lse = np.zeros((len(r), Bq), dtype=np.float64)
    num = np.zeros((len(r), Bq, d), dtype=np.float64) if want_numden else None
    den = np.zeros((len(r), Bq), dtype=np.float64) if want_numden else None
    _check(_load().orc_ht_attention(_ptr(_bits(Q)), _ptr(_bits(K)), _ptr(_bits(V)), B, H, N, d,
                                    Bq, Bk, scale, _ptr(r), len(r), _ptr(counts), _ptr(idx),
                                    _ptr(lw), cap, int(nq_max or 0),
                                    nthreads or default_threads(), _ptr(O), _ptr(lse),
                                    _ptr(num), _ptr(den)), "ht_attention")
    if want_numden:
        return O, lse, num, den
    return O, lse


def forward(Q, K, V, shape, rows, C, iters, budget_bp, seed, Bq=128, Bk=16, scale=None,
            nthreads=None, batch_offset=0, head_offset=0):
    """Whole path for the listed rows.  Returns dict(p32, counts, idx, logw, O).

    batch_offset, head_offset: global index of the tensors' first batch
    element and head when they are a slice of a larger problem."""
    B, H, N, d = shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    nK = -(-N // Bk)
    r = _rows(rows)
    p32 = np.zeros((len(r), nK), dtype=np.float32)
    counts = np.zeros(len(r), dtype=np.int32)
    idx = np.full((len(r), nK), -1, dtype=np.int32)
    logw = np.zeros((len(r), nK), dtype=np.float32)
    O = np.zeros((len(r), Bq, d), dtype=np.float64)
    _check(_load().orc_forward(_ptr(_bits(Q)), _ptr(_bits(K)), _ptr(_bits(V)), B, H, N, d, Bq,
                               Bk, C, iters, int(budget_bp), scale, int(seed) & (2**64 - 1),
                               _ptr(r), len(r), nthreads or default_threads(), _ptr(p32),
                               _ptr(counts), _ptr(idx), _ptr(logw), _ptr(O), int(batch_offset),
                               int(head_offset)), "forward")
    return dict(p32=p32, counts=counts, idx=idx, logw=logw, O=O)
