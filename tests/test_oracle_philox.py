"""Pin: the oracle's Philox4x32-10 against cuRAND's host-side generator.

cuRAND's host PHILOX4_32_10 generator (run on the CPU, never read) emits
output word n as word (n mod 4) of Philox4x32-10 at counter
(q div 65536 as a 64-bit value split over words 0-1, q mod 65536, 0) with
q = n div 4 and key (seed lo, seed hi).  That layout was established by
experiment; it exercises counter words 0, 1, 2 and both key words.
"""
import ctypes
import os

import numpy as np
import pytest

import oracle

_CURAND = "/usr/local/cuda/lib64/libcurand.so"


def _curand_host(seed, offset, n):
    cr = ctypes.CDLL(_CURAND)
    gen = ctypes.c_void_p()
    assert cr.curandCreateGeneratorHost(ctypes.byref(gen), 161) == 0  # PHILOX4_32_10
    try:
        assert cr.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        assert cr.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(offset)) == 0
        out = np.zeros(n, dtype=np.uint32)
        assert cr.curandGenerate(gen, out.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(n)) == 0
        return out
    finally:
        cr.curandDestroyGenerator(gen)


@pytest.mark.skipif(not os.path.exists(_CURAND), reason="libcurand not present")
@pytest.mark.parametrize("seed", [0, 1, 0x0123456789ABCDEF, 2**64 - 1])
@pytest.mark.parametrize("offset", [0, 4 * 65536 * 3 + 4 * 17, 2**50 + 4 * 65536 * 5, 2**62])
def test_philox_matches_curand_host(seed, offset):
    n = 64
    out = _curand_host(seed, offset, n)
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for m in range(n):
        pos = offset + m
        q = pos // 4
        hi = q // 65536
        ctr = [hi & 0xFFFFFFFF, hi >> 32, q % 65536, 0]
        w = oracle.philox4x32_10(ctr, key)
        assert int(w[pos % 4]) == int(out[m]), (seed, offset, m)


def test_philox_counter_words_all_matter():
    """Each counter and key word changes the output (no word is ignored)."""
    base = oracle.philox4x32_10([1, 2, 3, 4], [5, 6])
    for k in range(4):
        c = [1, 2, 3, 4]
        c[k] ^= 1
        assert not np.array_equal(oracle.philox4x32_10(c, [5, 6]), base)
    for k in range(2):
        key = [5, 6]
        key[k] ^= 1
        assert not np.array_equal(oracle.philox4x32_10([1, 2, 3, 4], key), base)


GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "philox4x32_10_kat.txt")


def _kat():
    rows = []
    for line in open(GOLDEN):
        if line.strip() and not line.startswith("#"):
            w = [int(x, 16) for x in line.split()]
            rows.append((w[0:4], w[4:6], w[6:10]))
    return rows


@pytest.mark.parametrize("ctr,key,out", _kat())
def test_philox_known_answer_vectors(ctr, key, out):
    """The published known-answer vectors set every counter word, including
    word 3 (the sampler's batch index), which cuRAND's host generator above
    never sets."""
    assert [int(x) for x in oracle.philox4x32_10(ctr, key)] == out
