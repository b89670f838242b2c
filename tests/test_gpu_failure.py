"""Failure detection on the GPU without a GPU fault.

Every wait of the scoring and attention kernels on an mbarrier is bounded.
These tests shorten the bound to a few milliseconds and make the copy
producer stop after its first tile (test hooks of the library), so the waits
for the later tiles run out for real: the call must return, the workspace
status word must carry ABATT_DEVFLAG_TIMEOUT, and a normal call on the same
stream afterwards must give exactly what it gave before (the CTAs drained
their copies and MMAs and freed tensor memory).  Nothing traps and no wait is
unbounded.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_20_b200 import abatt, synth

pytestmark = pytest.mark.gpu

WAIT_NS = 5_000_000  # 5 ms


class _Stalled:
    """Short waits and a stalled producer, restored on exit."""

    def __init__(self, mask):
        self.mask = mask

    def __enter__(self):
        abatt.test_set(abatt.TEST_WAIT_NS, WAIT_NS)
        abatt.test_set(abatt.TEST_STALL, self.mask)

    def __exit__(self, *exc):
        abatt.test_set(abatt.TEST_STALL, 0)
        abatt.test_set(abatt.TEST_WAIT_NS, 0)


def test_attention_wait_runs_out_and_the_next_call_is_exact():
    shape = (1, 2, 4096, 128)
    Bk = 16
    Q, K, V = (synth.random_bf16(shape, s).cuda() for s in (51, 52, 53))
    rows = np.arange(2 * 32)
    p = synth.random_probs(len(rows), 256, 54, 0.3)
    c, i, lw, _, _ = oracle.sample(p, shape, rows, 2500, 54, Bk=Bk)
    assert c.min() > 2 * 128 // Bk  # every row has several tiles: every CTA stalls
    counts, idx, logw = (torch.from_numpy(x).cuda() for x in (c, i, lw))
    cfg = abatt.Config(kv_block=Bk)
    ws = torch.empty(abatt.workspace_size(abatt.CALL_ATTENTION, shape, cfg), dtype=torch.uint8, device="cuda")
    before = abatt.attention(Q, K, V, counts, idx, logw, cfg, workspace=ws)
    torch.cuda.synchronize()
    assert abatt.read_status(ws) == 0
    with _Stalled(abatt.TEST_STALL_ATTENTION):
        abatt.attention(Q, K, V, counts, idx, logw, cfg, workspace=ws)
        torch.cuda.synchronize()  # the call returns
        assert abatt.read_status(ws) & abatt.DEVFLAG_TIMEOUT
    after = abatt.attention(Q, K, V, counts, idx, logw, cfg, workspace=ws)
    torch.cuda.synchronize()
    assert abatt.read_status(ws) == 0
    assert torch.equal(after, before)
    ref, _ = oracle.ht_attention(Q.cpu(), K.cpu(), V.cpu(), shape, rows, c, i, lw, Bk=Bk)
    got = after.float().cpu().numpy().reshape(2, 32, 128, 128).reshape(64, 128, 128)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 5e-3


def test_scoring_wait_runs_out_and_the_next_call_is_exact():
    w = synth.TINY
    Q, K, _ = (t.cuda() for t in synth.generate(w))
    cfg = abatt.Config(kv_block=w.Bk, clusters=w.clusters, kmeans_iters=w.iters)
    ws = torch.empty(abatt.workspace_size(abatt.CALL_SELECT, w.shape, cfg), dtype=torch.uint8, device="cuda")
    before = abatt.select(Q, K, cfg, workspace=ws)
    torch.cuda.synchronize()
    assert abatt.read_status(ws) == 0
    with _Stalled(abatt.TEST_STALL_SCORE):
        abatt.select(Q, K, cfg, workspace=ws)
        torch.cuda.synchronize()
        assert abatt.read_status(ws) & abatt.DEVFLAG_TIMEOUT
    after = abatt.select(Q, K, cfg, workspace=ws)
    torch.cuda.synchronize()
    assert abatt.read_status(ws) == 0
    assert torch.equal(after, before)


@pytest.mark.parametrize("deg,bound", [(3, 8.6e-5), (4, 2.9e-6)])
def test_fma_pipe_exp2_against_exp2f_and_float64(deg, bound):
    # the polynomial's fitted relative error (exact arithmetic) plus a few
    # fp32 roundings of its evaluation
    tol = bound + 8 * 2.0**-24
    x = torch.linspace(-126.0, 0.0, 2**22 + 1, dtype=torch.float64).float()
    y = abatt.test_exp2_poly(x.cuda(), deg).cpu().double()
    ref = torch.exp2(x.double())
    assert float(((y - ref).abs() / ref).max()) <= tol
    # against CUDA's exp2f (torch.exp2 on a CUDA float tensor)
    y32 = torch.exp2(x.cuda()).cpu().double()
    assert float(((y - y32).abs() / y32).max()) <= tol + 2.0**-22
    # integers are exact powers of two (f = 0 leaves the constant term 1)
    n = torch.arange(-126, 1, dtype=torch.float32)
    assert torch.equal(abatt.test_exp2_poly(n.cuda(), deg).cpu(), torch.exp2(n.double()).float())
    # at and below -127 (and -inf) the result is +0
    z = abatt.test_exp2_poly(torch.tensor([-127.0, -127.5, -300.0, float("-inf")], device="cuda"), deg).cpu()
    assert torch.equal(z.view(torch.int32), torch.zeros(4, dtype=torch.int32))
