"""The allocation-free attention entry point (abatt_attention_noalloc).

Some callers cannot allocate device memory at call time (they run inside a
memory pool they do not own, or their host forbids allocation on the
inference path).  For them the library offers one attention call whose
scratch lives in a fixed array inside the library.  These checks call it
through the C ABI and compare it with the regular abatt_attention on the same
inputs, twice in a row (the second call reuses the scratch the first left
behind): the two calls run the same kernels on the same inputs, so O and lse
must be bit for bit the same.  Around the second call the device's free
memory must not change, and oversized problems are refused before any launch.

This file is collected last on purpose, and passes both alone and after the
other GPU tests.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_20_b200 import abatt, synth

pytestmark = pytest.mark.gpu


def _lists(shape, Bk, bp, seed):
    B, H, N, d = shape
    nK = -(-N // Bk)
    rows = np.arange(B * H * (-(-N // 128)))
    p = synth.random_probs(len(rows), nK, seed, 0.3)
    c, i, lw, _, _ = oracle.sample(p, shape, rows, bp, seed, Bk=Bk)
    return (torch.from_numpy(c).cuda(), torch.from_numpy(i).cuda(), torch.from_numpy(lw).cuda())


@pytest.mark.parametrize("shape,Bk", [((1, 2, 4096, 64), 16), ((2, 3, 1000, 128), 32)])
def test_noalloc_matches_attention_twice(shape, Bk):
    Q, K, V = (synth.random_bf16(shape, s).cuda() for s in (91, 92, 93))
    counts, idx, logw = _lists(shape, Bk, 1500, 94)
    cfg = abatt.Config(kv_block=Bk)
    ref, ref_lse = abatt.attention(Q, K, V, counts, idx, logw, cfg, want_lse=True)
    status = torch.full((1,), 0x5A5A, dtype=torch.int32, device="cuda")
    outs = [torch.empty_like(Q) for _ in range(2)]
    lses = [torch.empty(shape[:3], dtype=torch.float32, device="cuda") for _ in range(2)]
    for k in range(2):
        outs[k].fill_(float("nan"))
        lses[k].fill_(float("nan"))
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        abatt.attention_noalloc(Q, K, V, counts, idx, logw, cfg, out=outs[k], lse=lses[k], dev_status=status)
        torch.cuda.synchronize()
        free1 = torch.cuda.mem_get_info()[0]
        if k == 1:  # the first call may load the module's image; the second allocates nothing
            assert free1 == free0
        assert int(status.item()) == 0
        assert torch.equal(outs[k], ref)
        assert torch.equal(lses[k].view(torch.int32), ref_lse.view(torch.int32))
    # and it is the method's attention: rows of the output against the float64 oracle
    B, H, N, d = shape
    nQ = -(-N // 128)
    rows = np.array([0, nQ - 1, B * H * nQ - 1])
    c, i, lw = (t.cpu().numpy() for t in (counts, idx, logw))
    o5, _ = oracle.ht_attention(Q.cpu(), K.cpu(), V.cpu(), shape, rows, c[rows], i[rows], lw[rows], Bk=Bk)
    got = np.zeros_like(o5)
    Of = outs[1].float().cpu().numpy()
    for k, r in enumerate(rows):
        bh, q = divmod(int(r), nQ)
        n = min(128, N - q * 128)
        got[k, :n] = Of[bh // H, bh % H, q * 128:q * 128 + n]
    assert np.linalg.norm(got - o5) / np.linalg.norm(o5) <= 5e-3
    assert np.max(np.abs(got - o5)) <= 2e-2


def test_noalloc_status_reads_pending_until_the_call_completes():
    # on a call that the host refuses after the argument checks nothing is
    # launched; on a completed call the word holds the call's flags (here 0)
    shape = (1, 1, 512, 64)
    Q, K, V = (synth.random_bf16(shape, s).cuda() for s in (1, 2, 3))
    counts, idx, logw = _lists(shape, 16, 2000, 5)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(Q)
    abatt.attention_noalloc(Q, K, V, counts, idx, logw, abatt.Config(kv_block=16), out=out, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    with pytest.raises(ValueError):  # the binding checks the output buffer
        abatt.attention_noalloc(Q, K, V, counts, idx, logw, abatt.Config(kv_block=16), out=out[:, :, :256])


def test_noalloc_refuses_shapes_beyond_its_scratch():
    cfg = abatt.Config(kv_block=16)
    big = (1, 40, 75600, 128)  # needs far more than the fixed scratch
    assert abatt.workspace_size(abatt.CALL_ATTENTION, big, cfg) > abatt.NOALLOC_SCRATCH_BYTES
    sh = abatt._Shape(*big)
    one = torch.zeros(1, dtype=torch.int32, device="cuda")  # never read: refused on the host
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    code = abatt.lib().abatt_attention_noalloc(
        abatt._ptr(x), abatt._ptr(x), abatt._ptr(x), abatt.ctypes.byref(sh),
        abatt.ctypes.byref(cfg._c(128)), abatt._ptr(one), abatt._ptr(one), abatt._ptr(one), 1,
        abatt._ptr(x), None, None, None)
    assert code == 2  # ABATT_ERR_UNSUPPORTED
