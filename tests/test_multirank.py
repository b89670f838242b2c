"""The N > 1 path of bench.py on CPU: two ranks over gloo.

Each rank runs bench.py's host-side pieces (its share of the job, the
max-over-ranks reduction of the timed region, the whole-job value) and the
parent checks what every rank got.  No GPU: the ranks exchange plain tensors.
"""
import datetime
import os
import socket

import numpy as np
import pytest

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, queue):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from block_sparse_attention_20_b200 import synth

        w = synth.WAN_14B
        plan = bench.rank_plan(w, rank, world)
        # each rank's own timed region: the job time is the slowest rank's
        t = bench.max_over_ranks(3.0 + 2.0 * rank, world)
        v = bench.job_value(1.0e12, world, t)
        # each rank draws its own inputs (a small case keeps this quick)
        tiny = synth.TINY.with_(seed=plan["data_seed"])
        q = synth.generate(tiny, heads=1)[0].float().numpy()
        queue.put((rank, plan, t, v, float(q[0, 0, :8, 0].sum())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_share_the_job_and_take_the_slowest_time():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, WORLD, port, queue)) for r in range(WORLD)]
    for p in procs:
        p.start()
    try:
        got = sorted(queue.get(timeout=120) for _ in range(WORLD))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    (r0, plan0, t0, v0, q0), (r1, plan1, t1, v1, q1) = got
    assert (r0, r1) == (0, 1)
    # disjoint batch elements, one Philox key, different inputs
    assert plan0["batch_offset"] == 0 and plan1["batch_offset"] == 1
    assert plan0["philox_seed"] == plan1["philox_seed"]
    assert plan0["data_seed"] != plan1["data_seed"] and q0 != q1
    # both ranks report the slowest rank's time and the whole job's value
    assert t0 == t1 == 5.0
    assert v0 == v1 == pytest.approx(1.0e12 * WORLD / 5e-3 / 1e12)


def test_rank_plan_rejects_a_rank_outside_the_world():
    import bench
    from block_sparse_attention_20_b200 import synth

    with pytest.raises(ValueError):
        bench.rank_plan(synth.WAN_14B, 2, 2)
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert np.isclose(bench.job_value(2e12, 1, 1000.0), 2.0)


def _heads_rank_main(rank, world, port, queue):
    """One rank of the head split: its heads of the one tiny problem, drawn
    through the oracle with the rank's head offset."""
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        from block_sparse_attention_20_b200 import synth

        w = synth.TINY
        plan = bench.rank_plan(w, rank, world, "heads")
        (Q, K, V), wr = bench.rank_inputs(w, plan)
        rows = np.arange(wr.rows)
        out = oracle.forward(Q, K, V, wr.shape, rows, w.clusters, w.iters, w.budget_bp, w.seed, Bk=w.Bk,
                             nthreads=2, head_offset=plan["head_offset"])
        mine = {"heads": (plan["head_offset"], plan["heads"]), "counts": out["counts"].tolist(),
                "idx": [out["idx"][k, :out["counts"][k]].tolist() for k in range(len(rows))]}
        got = [None] * world
        dist.all_gather_object(got, mine)
        if rank == 0:
            queue.put(got)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_head_split_draws_exactly_what_one_call_draws():
    # two gloo ranks each take one head of the tiny problem; together they
    # cover every head once, and their lists are the lists of one pass over
    # the whole problem (the sampler's counter carries the global head)
    import torch.multiprocessing as mp

    import oracle
    from block_sparse_attention_20_b200 import synth

    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_heads_rank_main, args=(r, WORLD, port, queue)) for r in range(WORLD)]
    for p in procs:
        p.start()
    try:
        got = queue.get(timeout=300)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    w = synth.TINY
    Q, K, V = synth.generate(w)
    whole = oracle.forward(Q, K, V, w.shape, np.arange(w.rows), w.clusters, w.iters, w.budget_bp, w.seed,
                           Bk=w.Bk, nthreads=2)
    heads = []
    for part in got:
        h0, nh = part["heads"]
        heads += list(range(h0, h0 + nh))
        for k in range(nh * w.nQ):
            r = h0 * w.nQ + k
            assert part["counts"][k] == whole["counts"][r]
            assert part["idx"][k] == whole["idx"][r, :whole["counts"][r]].tolist()
    assert heads == list(range(w.H))
