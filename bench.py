"""Benchmark of the AB-Attention hot path on B200.

One step = one pass of the whole path (IBCS selector -> SIP sampler -> gather
attention) over one batch of the synthetic Wan2.1-14B-720p-shaped workload
(75,600 tokens, 40 heads, d = 128, 8 % block budget = 92 % skip).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl abatt|reference]

Prints one JSON line (rank 0).  `value` is dense-equivalent TFLOPS
(4 B H N^2 d per step / step time) summed over ranks; the roofline object
covers the gather-attention kernel (executed 128x128 tiles, tensor bound).
With N > 1 GPUs (torchrun), every rank runs its own batch element (heads are
independent; no collective on the data path): weak scaling; with
`--split heads` the ranks share out the heads of the one problem instead
(strong scaling).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_20_b200 import synth  # noqa: E402

METRIC = "attention ms & dense-equiv TFLOPS at 90% skip; % bf16 tensor peak (1 B200)"
FALLBACK_PEAK_TFLOPS = 1590.0


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="abatt", choices=["abatt", "reference"])
    ap.add_argument("--workload", default="wan14b-720p", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--sweep", action="store_true",
                    help="the sweep workloads (H=24, N x budget x Bk): one JSON line per point, then a table")
    ap.add_argument("--sweep-n", default=None, help="comma-separated subset of the sweep's N")
    ap.add_argument("--budget-bp", type=int, default=None, help="override (10000 = keep-all)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-keep-all", action="store_true", help="skip the keep-all attention timing")
    ap.add_argument("--e2e-heads", type=int, default=2, help="heads per chunk of the host pipeline")
    ap.add_argument("--selection", default="sip", choices=["sip", "topk"],
                    help="sip: the method's draw; topk: the truncating baseline")
    ap.add_argument("--draws", default="independent", choices=["independent", "paired"],
                    help="paired: query blocks 2j, 2j+1 share the sampler's uniforms")
    ap.add_argument("--scoring", default="keys", choices=["keys", "block-means"],
                    help="keys: every key scored (the method); block-means: the coarse baseline")
    ap.add_argument("--split", default="batch", choices=["batch", "heads"],
                    help="N > 1: batch -- one batch element per GPU (weak scaling); heads -- the "
                         "heads of one problem shared out over the GPUs (strong scaling)")
    return ap.parse_args(argv)


def attention_source(csrc: str) -> bytes:
    """The source the gather-attention kernel is compiled from."""
    head = open(os.path.join(csrc, "kernels.cuh"), "rb").read()
    cut = head.find(b"// ---- gather attention")
    return b"".join(open(os.path.join(csrc, f), "rb").read() for f in ("attention.cu", "common.cuh")) + \
        (head[cut:] if cut >= 0 else head)


TRAFFIC_KEY = os.path.join(ROOT, "profiles", "gather_attn_kernel.json")


def attention_traffic(rows: int, key_path: str = None):
    """DRAM bytes of one gather_attn_kernel launch from the committed ncu
    counters (profiles/gather_attn_kernel.json: bytes per query block, scaled
    by the launch's query blocks -- the kernel's DRAM traffic is its
    compulsory Q/K/V/O bytes, which grow with the query blocks).  None when
    the kernel source differs from the one the counters were taken on:
    attention.cu, common.cuh and the gather-attention part of kernels.cuh
    (from its "---- gather attention" heading on)."""
    import hashlib
    csrc = os.path.join(ROOT, "block_sparse_attention_20_b200", "csrc")
    try:
        src = attention_source(csrc)
        with open(key_path or TRAFFIC_KEY) as f:
            key = json.load(f)
    except (OSError, ValueError):
        return None
    if key.get("source_sha256_16") != hashlib.sha256(src).hexdigest()[:16]:
        return None
    return int(key["dram_bytes_per_query_block"]) * rows


def run_sweep(args):
    """Latency, tensor-pipe fraction and error of every sweep point (H=24,
    d=128; N x budget x Bk) on one GPU.  The error is the relative L2 of O
    against the same kernel in keep-all mode (budget 100 %: every block,
    weight 1 -- dense attention, checked against the float64 oracle by the
    GPU tests).  Inputs are drawn on the GPU (synth.generate_on_device)."""
    import torch

    from block_sparse_attention_20_b200 import abatt

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    pk, src = peaks()
    peak = pk.get("bf16_tflops", FALLBACK_PEAK_TFLOPS)
    Ns = synth.SWEEP_N if not args.sweep_n else tuple(int(x) for x in args.sweep_n.split(","))
    reps = max(3, min(args.steps, 10))  # per sweep point
    stream = torch.cuda.current_stream()
    table = []
    for N in Ns:
        w0 = synth.sweep(N, 100, 16)
        Q, K, V = synth.generate_on_device(w0, dev)
        shape = w0.shape
        for Bk in synth.SWEEP_BK:
            O_ref = None
            for bpct in sorted(synth.SWEEP_BUDGET, reverse=True):  # keep-all first: the reference
                w = synth.sweep(N, bpct, Bk)
                cfg = abatt.Config(kv_block=Bk, clusters=w.clusters, kmeans_iters=w.iters,
                                   budget_bp=w.budget_bp, seed=w.seed)
                rows, nK = w.rows, w.nK
                p = torch.empty((rows, nK), dtype=torch.float32, device=dev)
                counts = torch.empty(rows, dtype=torch.int32, device=dev)
                idx = torch.empty((rows, nK), dtype=torch.int32, device=dev)
                logw = torch.empty((rows, nK), dtype=torch.float32, device=dev)
                O = torch.empty_like(Q)
                ws_sel = torch.empty(abatt.workspace_size(abatt.CALL_SELECT, shape, cfg), dtype=torch.uint8,
                                     device=dev)
                ws_small = torch.empty(256, dtype=torch.uint8, device=dev)
                ws_att = torch.empty(abatt.workspace_size(abatt.CALL_ATTENTION, shape, cfg),
                                     dtype=torch.uint8, device=dev)
                ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(reps)]
                for k in range(reps + 2):
                    e = ev[k - 2] if k >= 2 else None
                    if e: e[0].record(stream)
                    abatt.select(Q, K, cfg, p=p, workspace=ws_sel, stream=stream)
                    if e: e[1].record(stream)
                    abatt.sample(p, shape, cfg, out=(counts, idx, logw), workspace=ws_small, stream=stream)
                    if e: e[2].record(stream)
                    abatt.attention(Q, K, V, counts, idx, logw, cfg, out=O, workspace=ws_att, stream=stream)
                    if e: e[3].record(stream)
                torch.cuda.synchronize()
                status = abatt.read_status(ws_small) | abatt.read_status(ws_sel) | abatt.read_status(ws_att)
                sel = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
                smp = statistics.median(e[1].elapsed_time(e[2]) for e in ev)
                att = statistics.median(e[2].elapsed_time(e[3]) for e in ev)
                c = counts.cpu().numpy().astype(np.int64)
                bpt = 128 // Bk
                tiles = int(((c + bpt - 1) // bpt).sum())
                exec_tf = tiles * 4.0 * 128 * 128 * w.d / (att * 1e-3) / 1e12
                dense_flop = 4.0 * w.H * N * N * w.d
                skip = 1.0 - float(np.minimum(c * Bk, N).sum()) / (w.H * w.nQ * N)
                if O_ref is None:
                    O_ref = O.float()
                    err = 0.0
                else:
                    err = float((O.float() - O_ref).norm() / O_ref.norm())
                rec = {"N": N, "kv_block": Bk, "budget_pct": bpct, "select_ms": sel, "sample_ms": smp,
                       "attention_ms": att, "total_ms": sel + smp + att,
                       "dense_equiv_tflops": dense_flop / ((sel + smp + att) * 1e-3) / 1e12,
                       "executed_tflops_attention": exec_tf, "tensor_frac": exec_tf / peak,
                       "realized_skip": skip, "rel_l2_vs_keep_all": err, "device_status": status}
                print(json.dumps(rec), flush=True)
                table.append(rec)
                del p, counts, idx, logw, O, ws_sel, ws_att
            del O_ref
        del Q, K, V
        torch.cuda.empty_cache()
    print(f"\npeak {peak:.0f} TFLOP/s ({src} bf16 burst)")
    print("| N | Bk | budget | select ms | sample ms | attention ms | total ms | dense-equiv TFLOP/s "
          "| executed TFLOP/s | tensor frac | skip | rel L2 vs keep-all |")
    print("|---|---|---|---|---|---|---|---|---|---|---|---|")
    for r in table:
        print(f"| {r['N']} | {r['kv_block']} | {r['budget_pct']} % | {r['select_ms']:.2f} | {r['sample_ms']:.2f} "
              f"| {r['attention_ms']:.2f} | {r['total_ms']:.2f} | {r['dense_equiv_tflops']:.0f} "
              f"| {r['executed_tflops_attention']:.0f} | {r['tensor_frac']:.2f} | {r['realized_skip']:.3f} "
              f"| {r['rel_l2_vs_keep_all']:.3f} |")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return {"bf16_tflops": FALLBACK_PEAK_TFLOPS, "bf16_tflops_sustained": 1400.0,
                "hbm_gbs": 6650.0}, "fallback"


class Clocks:
    """nvidia-smi sampler running during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def bench_config(w, args) -> dict:
    """The workload description both arms print (same keys, same values)."""
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
            "budget_bp": w.budget_bp, "kv_block": w.Bk, "clusters": w.clusters,
            "kmeans_iters": w.iters, "selection": args.selection,
            "scoring": args.scoring, "draws": args.draws,
            "per_rank": ("heads [r*H/N, (r+1)*H/N) of one problem" if args.split == "heads"
                         else "one batch element per GPU"),
            "l2": "inputs (Q,K,V 2.3 GB) exceed the 126 MB L2; no flush"}


def run_reference(args, w):
    """The tier's reference arm: the float64 CPU oracle, as it stands, on a
    bounded sample of query blocks per step (every k-th row).  `value` is the
    dense-equivalent throughput of the whole workload at the measured rate
    (the measured time per sampled row times the workload's rows); the timed
    region itself is `ms_per_step` x `steps`."""
    import oracle

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    if args.selection != "sip" or args.scoring != "keys" or args.draws != "independent":
        print(json.dumps({"impl": "reference", "unavailable":
                          "the oracle's forward pass covers the method's own sampler and scoring only"}))
        return
    cores = oracle.default_threads()
    Q, K, V = synth.generate(w)
    nrows = max(8, min(cores, 64))
    stride = max(1, w.rows // nrows)
    rows = np.arange(0, w.rows, stride)[:nrows]

    def step():
        oracle.forward(Q, K, V, w.shape, rows, w.clusters, w.iters, w.budget_bp, w.seed, Bk=w.Bk,
                       nthreads=cores)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps  # measured seconds per step (the sample)
    scale = w.rows / len(rows)
    full = dt * scale  # the whole workload at the measured rate
    dense = 4.0 * w.B * w.H * w.N * w.N * w.d
    value = dense / full / 1e12
    sample = (f"{len(rows)} of {w.rows} query blocks per step (every {stride}th); value scales the "
              f"measured time x{scale:.1f} to the whole workload")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS (dense-equivalent)",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w, args),
        "extrapolated_ms_per_workload": full * 1e3,
        "rows_per_step": int(len(rows)),
        "cpu_baseline": {"value": value, "unit": "TFLOPS (dense-equivalent)", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS (dense-equivalent)", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(w, Q, K, V):
    """The oracle on this host's cores, on a bounded sample of the workload:
    the whole path (k-means, block probabilities, draw, weighted attention)
    and, separately, dense float64 attention on the same query blocks."""
    import oracle

    cores = oracle.default_threads()
    nrows = max(4, min(16 * cores, w.rows))
    stride = max(1, w.rows // nrows)
    rows = np.arange(0, w.rows, stride)[:nrows]
    t0 = time.perf_counter()
    oracle.forward(Q, K, V, w.shape, rows, w.clusters, w.iters, w.budget_bp, w.seed, Bk=w.Bk,
                   nthreads=cores)
    dt = time.perf_counter() - t0
    full = dt * w.rows / len(rows)
    dense = 4.0 * w.B * w.H * w.N * w.N * w.d
    # dense attention (O1) on a quarter of the same rows
    drows = rows[::4]
    t0 = time.perf_counter()
    oracle.dense_attention(Q, K, V, w.shape, drows, nthreads=cores)
    dt_dense = time.perf_counter() - t0
    full_dense = dt_dense * w.rows / len(drows)
    # and the whole tiny workload (every query block) on one thread
    tw = synth.TINY
    Qt, Kt, Vt = synth.generate(tw)
    t0 = time.perf_counter()
    oracle.forward(Qt, Kt, Vt, tw.shape, np.arange(tw.rows), tw.clusters, tw.iters, tw.budget_bp, tw.seed,
                   Bk=tw.Bk, nthreads=1)
    dt1 = time.perf_counter() - t0
    return {"value": dense / full / 1e12, "unit": "TFLOPS (dense-equivalent)", "cores": cores,
            "kind": "oracle",
            "sample": f"{len(rows)} of {w.rows} query blocks (every {stride}th), {dt:.1f} s, "
                      f"extrapolated x{w.rows / len(rows):.1f}",
            "dense_attention": {"value": dense / full_dense / 1e12, "unit": "TFLOPS",
                                "sample": f"{len(drows)} query blocks, {dt_dense:.1f} s, "
                                          f"extrapolated x{w.rows / len(drows):.1f}",
                                "extrapolated_s": full_dense},
            "tiny_one_thread_s": dt1}


def rank_plan(w, rank: int, world: int, split: str = "batch") -> dict:
    """What rank `rank` of `world` computes; no collective on the data path.

    split="batch" (weak scaling): batch elements [rank*B, (rank+1)*B) of a
    world*B-element problem, inputs drawn with data seed w.seed + rank, the
    sampler on the global batch index (batch_offset) with the job's one
    Philox key.
    split="heads" (strong scaling): heads [rank*H//world, (rank+1)*H//world)
    of the one problem (data seed w.seed), the sampler on the global head
    index (head_offset), so the job draws exactly what one call over all
    heads draws."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world {world}")
    if split == "batch":
        return {"batch_offset": rank * w.B, "head_offset": 0, "heads": w.H, "data_seed": w.seed + rank,
                "philox_seed": w.seed}
    if split == "heads":
        if world > w.B * w.H:
            raise ValueError(f"{world} ranks for {w.B * w.H} heads")
        if w.B != 1:
            raise ValueError("the head split shares out the heads of one batch element")
        h0, h1 = rank * w.H // world, (rank + 1) * w.H // world
        return {"batch_offset": 0, "head_offset": h0, "heads": h1 - h0, "data_seed": w.seed,
                "philox_seed": w.seed}
    raise ValueError(f"unknown split {split!r}")


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The slowest rank's time (every rank takes part; returns x when alone)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(flop_per_rank: float, world: int, ms: float) -> float:
    """Whole-job dense-equivalent TFLOPS: the work of all ranks over the
    slowest rank's time."""
    return flop_per_rank * world / (ms * 1e-3) / 1e12


def rank_inputs(w, plan):
    """This rank's Q, K, V (CPU bf16) and its share of the workload."""
    if plan["heads"] == w.H and plan["head_offset"] == 0:
        return synth.generate(w.with_(seed=plan["data_seed"])), w
    Q, K, V = synth.generate(w.with_(seed=plan["data_seed"]))
    h0, h1 = plan["head_offset"], plan["head_offset"] + plan["heads"]
    return tuple(t[:, h0:h1].contiguous() for t in (Q, K, V)), w.with_(H=h1 - h0)


def roofline_peaks(pk: dict, sm_mhz):
    """(burst peak, peak scaled to the sampled SM clock) in TFLOP/s.

    The burst figure is cuBLAS bf16 timed alone; the sustained figure was
    measured at the median clock recorded beside it, so scaling it by the
    clock this run saw gives the peak at this run's clock."""
    burst = float(pk.get("bf16_tflops", FALLBACK_PEAK_TFLOPS))
    sus = pk.get("bf16_tflops_sustained")
    mhz = (pk.get("clocks_under_load") or {}).get("sm_mhz_median")
    scaled = float(sus) * float(sm_mhz) / float(mhz) if sus and mhz and sm_mhz else None
    return burst, scaled


def main():
    args = parse()
    w = synth.WORKLOADS[args.workload]
    if args.budget_bp is not None:
        w = w.with_(budget_bp=args.budget_bp)
    if args.impl == "reference":
        run_reference(args, w)
        return
    if args.sweep:
        run_sweep(args)
        return

    import torch
    import torch.distributed as dist

    from block_sparse_attention_20_b200 import abatt

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    plan = rank_plan(w, rank, world, args.split)
    (Qc, Kc, Vc), wr = rank_inputs(w, plan)
    Q, K, V = Qc.to(dev), Kc.to(dev), Vc.to(dev)
    shape = wr.shape
    cfg = abatt.Config(kv_block=w.Bk, clusters=w.clusters, kmeans_iters=w.iters,
                       budget_bp=w.budget_bp, seed=plan["philox_seed"],
                       batch_offset=plan["batch_offset"], head_offset=plan["head_offset"],
                       selection=abatt.SELECT_TOPK if args.selection == "topk" else abatt.SELECT_SIP,
                       scoring=(abatt.SCORE_BLOCK_MEANS if args.scoring == "block-means"
                                else abatt.SCORE_KEYS),
                       draws=abatt.DRAWS_PAIRED if args.draws == "paired" else abatt.DRAWS_INDEPENDENT)
    rows, nK = wr.rows, wr.nK
    p = torch.empty((rows, nK), dtype=torch.float32, device=dev)
    counts = torch.empty(rows, dtype=torch.int32, device=dev)
    idx = torch.empty((rows, nK), dtype=torch.int32, device=dev)
    logw = torch.empty((rows, nK), dtype=torch.float32, device=dev)
    O = torch.empty_like(Q)
    ws_sel = torch.empty(abatt.workspace_size(abatt.CALL_SELECT, shape, cfg), dtype=torch.uint8,
                         device=dev)
    ws_small = torch.empty(256, dtype=torch.uint8, device=dev)
    ws_att = torch.empty(abatt.workspace_size(abatt.CALL_ATTENTION, shape, cfg), dtype=torch.uint8,
                         device=dev)
    stream = torch.cuda.current_stream()

    # events: select | sample | pair segments | gather attention
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]

    def step(e=None):
        if e: e[0].record(stream)
        abatt.select(Q, K, cfg, p=p, workspace=ws_sel, stream=stream)
        if e: e[1].record(stream)
        abatt.sample(p, shape, cfg, out=(counts, idx, logw), workspace=ws_small, stream=stream)
        if e: e[2].record(stream)
        abatt.attention_plan(shape, counts, idx, logw, cfg, workspace=ws_att, stream=stream)
        if e: e[3].record(stream)
        abatt.attention_planned(Q, K, V, cfg, workspace=ws_att, out=O, stream=stream)
        if e: e[4].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with Clocks(local) as clk:
        time.sleep(0.3)  # let the sampler start before the timed region
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for k in range(args.steps):
            step(ev[k])
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    total_ms = max_over_ranks(start.elapsed_time(end), world, dev)
    med = lambda a, b: statistics.median(e[a].elapsed_time(e[b]) for e in ev)
    sel_ms, smp_ms, plan_ms, gat_ms = med(0, 1), med(1, 2), med(2, 3), med(3, 4)
    att_ms = med(2, 4)
    gat_mean = sum(e[3].elapsed_time(e[4]) for e in ev) / len(ev)
    ms_step = total_ms / args.steps
    status = abatt.read_status(ws_small) | abatt.read_status(ws_sel) | abatt.read_status(ws_att)

    c = counts.cpu().numpy().astype(np.int64)
    idx_h = idx.cpu().numpy()
    bpt = 128 // w.Bk
    # executed tiles: every row runs its own drawn blocks, 128/Bk per tile
    # (pairs of neighbouring rows share the gathers of common tiles, not the math)
    last = wr.nK - 1
    tail = wr.N - last * wr.Bk
    keys = np.zeros(rows, dtype=np.int64)
    for r in range(rows):
        L = c[r]
        keys[r] = L * wr.Bk - (wr.Bk - tail if L and idx_h[r, :L][-1] == last else 0)
    tiles = int(((c + bpt - 1) // bpt).sum())
    exec_flop = tiles * 4.0 * 128 * 128 * wr.d
    # algorithmic work: valid query rows x valid drawn keys
    nrows_q = np.minimum(128, wr.N - (np.arange(rows) % wr.nQ) * 128)
    alg_flop = float((4.0 * wr.d * nrows_q * keys).sum())
    rank_dense = 4.0 * wr.B * wr.H * wr.N * wr.N * wr.d
    job_dense = 4.0 * w.B * w.H * w.N * w.N * w.d * (world if args.split == "batch" else 1)
    skip = 1.0 - float((nrows_q * keys).sum()) / (wr.B * wr.H * wr.N * float(wr.N))

    pk, src = peaks()
    clocks = clk.summary()
    burst, at_clock = roofline_peaks(pk, clocks.get("sm_mhz"))
    achieved = alg_flop / (gat_mean * 1e-3) / 1e12
    # blocks the two rows of a pair both drew (gathered once for both), over
    # the blocks either drew
    both = either = 0
    for r in range(0, rows - 1, 2):
        if (r % wr.nQ) % 2 or r // wr.nQ != (r + 1) // wr.nQ:
            continue
        a0, a1 = idx_h[r, :c[r]], idx_h[r + 1, :c[r + 1]]
        k = np.intersect1d(a0, a1, assume_unique=True).size
        both += k
        either += a0.size + a1.size - k

    line = {
        "metric": METRIC,
        "value": job_value(job_dense, 1, ms_step),
        "unit": "TFLOPS (dense-equivalent)",
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak" if args.split == "batch" else "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": bench_config(w, args),
        "stages_ms": {"select": sel_ms, "sample": smp_ms, "attention": att_ms,
                      "attention_pair_segments": plan_ms, "attention_gather_kernel": gat_ms},
        "attention_ms": att_ms,
        "selector_sampler_share": (sel_ms + smp_ms) / (sel_ms + smp_ms + att_ms),
        "realized_skip": skip,
        "pair_shared_fraction": both / max(either, 1),
        "executed_tflops_attention": exec_flop / (gat_mean * 1e-3) / 1e12,
        "algorithmic_tflops_attention": achieved,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                     "frac": achieved / burst, "traffic": attention_traffic(rows),
                     "kernel": "gather_attn_kernel (timed alone, CUDA events on its stream)",
                     "flops": "algorithmic (valid query rows x drawn keys)",
                     "peak_source": f"{src} bf16 burst",
                     "peak_at_sampled_clock": at_clock,
                     "frac_at_sampled_clock": achieved / at_clock if at_clock else None},
        "rank_dense_tflop": rank_dense / 1e12,
        "device_status": status,
        "gpu_launches": 7 * args.steps,
        "clocks": clocks,
    }

    if not args.no_keep_all:
        line["keep_all"] = keep_all(abatt, cfg, Q, K, V, wr, O, ws_att, stream)
    if not args.no_e2e:
        line["e2e"] = e2e(abatt, cfg, Qc, Kc, Vc, dev, wr, args, world, job_dense)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:  # the host baseline: one process alone
        line["cpu_baseline"] = cpu_baseline(w, Qc, Kc, Vc)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def keep_all(abatt, cfg, Q, K, V, w, O, ws, stream):
    """The same attention kernel fed every key block with weight 1 (dense
    attention through the gather path), timed the same way: the pair
    segments once, then the gather kernel alone."""
    import torch

    rows, nK = w.rows, w.nK
    counts = torch.full((rows,), nK, dtype=torch.int32, device=Q.device)
    idx = torch.arange(nK, dtype=torch.int32, device=Q.device).repeat(rows, 1)
    logw = torch.zeros((rows, nK), dtype=torch.float32, device=Q.device)
    abatt.attention_plan(w.shape, counts, idx, logw, cfg, workspace=ws, stream=stream)
    for _ in range(2):
        abatt.attention_planned(Q, K, V, cfg, workspace=ws, out=O, stream=stream)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    reps = 3
    a.record(stream)
    for _ in range(reps):
        abatt.attention_planned(Q, K, V, cfg, workspace=ws, out=O, stream=stream)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    dense = 4.0 * w.B * w.H * w.N * w.N * w.d
    tiles = rows * ((nK + 128 // w.Bk - 1) // (128 // w.Bk))
    return {"gather_kernel_ms": ms, "dense_tflops": dense / (ms * 1e-3) / 1e12,
            "executed_tflops": tiles * 4.0 * 128 * 128 * w.d / (ms * 1e-3) / 1e12}


def e2e(abatt, cfg, Qc, Kc, Vc, dev, w, args, world, job_dense):
    """Same metric through the public host-to-host call: every step copies
    Q, K, V from pinned host memory to the device and O back, through
    abatt.HostPipeline (abatt_forward over chunks of heads, the copies of one
    chunk overlapped with the compute of the previous one).  `w` is this
    rank's share; `job_dense` the whole job's dense-equivalent FLOPs."""
    import torch
    import torch.distributed as dist

    hq, hk, hv = (t.pin_memory() for t in (Qc, Kc, Vc))
    ho = torch.empty_like(Qc).pin_memory()
    pipe = abatt.HostPipeline(w.shape, cfg, heads_per_chunk=args.e2e_heads, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        pipe(hq, hk, hv, ho)

    steps = max(3, args.steps // 4)
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / steps, world, dev)
    nbytes = Qc.numel() * 2
    return {"value": job_value(job_dense, 1, ms), "unit": "TFLOPS (dense-equivalent)",
            "ms_per_step": ms, "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
            "steps": steps, "heads_per_chunk": pipe.hc, "device_status": pipe.status()}


if __name__ == "__main__":
    main()
