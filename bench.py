"""Benchmark of the AB-Attention hot path on B200.

One step = one pass of the whole path (IBCS selector -> SIP sampler -> gather
attention) over one batch of the synthetic Wan2.1-14B-720p-shaped workload
(75,600 tokens, 40 heads, d = 128, 8 % block budget = 92 % skip).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl abatt|reference]

Prints one JSON line (rank 0).  `value` is dense-equivalent TFLOPS
(4 B H N^2 d per step / step time) summed over ranks; the roofline object
covers the gather-attention kernel (executed 128x128 tiles, tensor bound).
With N > 1 GPUs (torchrun), every rank runs its own batch element (heads are
independent; no collective on the data path): weak scaling.
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


def parse():
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
    return ap.parse_args()


def attention_source(csrc: str) -> bytes:
    """The source the gather-attention kernel is compiled from."""
    head = open(os.path.join(csrc, "kernels.cuh"), "rb").read()
    cut = head.find(b"// ---- gather attention")
    return b"".join(open(os.path.join(csrc, f), "rb").read() for f in ("attention.cu", "common.cuh")) + \
        (head[cut:] if cut >= 0 else head)


def attention_traffic(rows: int):
    """DRAM bytes of one gather_attn_kernel launch, from the committed ncu
    summary (bytes per query block, scaled by the launch's query blocks; DRAM
    traffic of the kernel is its compulsory Q/K/V/O bytes, which grow with the
    query blocks).  None when the kernel source differs from the one the
    counters were taken on: attention.cu, common.cuh and the gather-attention
    part of kernels.cuh (from its "---- gather attention" heading on)."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "block_sparse_attention_20_b200", "csrc")
    try:
        src = attention_source(csrc)
        txt = open(os.path.join(ROOT, "profiles", "gather_attn_kernel_wan1.3b.md")).read()
    except OSError:
        return None
    m = re.search(r"source sha256 ([0-9a-f]{16}); DRAM bytes per query block: ([0-9]+)", txt)
    if not m or m.group(1) != hashlib.sha256(src).hexdigest()[:16]:
        return None
    return int(m.group(2)) * rows


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


def run_reference(args, w):
    """The tier's reference arm: the float64 CPU oracle, as it stands, on a
    bounded sample of query blocks per step."""
    import oracle

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
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
    dt = (time.perf_counter() - t0) / args.steps
    full = dt * w.rows / len(rows)  # extrapolated to the whole workload
    dense = 4.0 * w.B * w.H * w.N * w.N * w.d
    value = dense / full / 1e12
    sample = f"{len(rows)} of {w.rows} query blocks per step (every {stride}th), time x{w.rows / len(rows):.1f}"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS (dense-equivalent)",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": full * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "budget_bp": w.budget_bp, "kv_block": w.Bk, "clusters": w.clusters},
        "cpu_baseline": {"value": value, "unit": "TFLOPS (dense-equivalent)", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS (dense-equivalent)", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(w, Q, K, V, budget_s=15.0):
    """The oracle on this host's cores, on a bounded sample of the workload."""
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
            "tiny_one_thread_s": dt1}


def rank_plan(w, rank: int, world: int) -> dict:
    """What rank `rank` of `world` computes (weak scaling, no collective on the
    data path): batch elements [rank*B, (rank+1)*B) of a world*B-element
    problem.  Its inputs are drawn with data seed w.seed + rank; its sampler
    uses the global batch index (batch_offset) with the job's one Philox key."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world {world}")
    return {"batch_offset": rank * w.B, "data_seed": w.seed + rank, "philox_seed": w.seed}


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

    plan = rank_plan(w, rank, world)
    Qc, Kc, Vc = synth.generate(w.with_(seed=plan["data_seed"]))
    Q, K, V = Qc.to(dev), Kc.to(dev), Vc.to(dev)
    shape = w.shape
    cfg = abatt.Config(kv_block=w.Bk, clusters=w.clusters, kmeans_iters=w.iters,
                       budget_bp=w.budget_bp, seed=plan["philox_seed"],
                       batch_offset=plan["batch_offset"],
                       selection=abatt.SELECT_TOPK if args.selection == "topk" else abatt.SELECT_SIP,
                       scoring=(abatt.SCORE_BLOCK_MEANS if args.scoring == "block-means"
                                else abatt.SCORE_KEYS),
                       draws=abatt.DRAWS_PAIRED if args.draws == "paired" else abatt.DRAWS_INDEPENDENT)
    rows, nK = w.rows, w.nK
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

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]

    def step(e=None):
        if e: e[0].record(stream)
        abatt.select(Q, K, cfg, p=p, workspace=ws_sel, stream=stream)
        if e: e[1].record(stream)
        abatt.sample(p, shape, cfg, out=(counts, idx, logw), workspace=ws_small, stream=stream)
        if e: e[2].record(stream)
        abatt.attention(Q, K, V, counts, idx, logw, cfg, out=O, workspace=ws_att, stream=stream)
        if e: e[3].record(stream)

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
    sel_ms = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    smp_ms = statistics.median(e[1].elapsed_time(e[2]) for e in ev)
    att_ms = statistics.median(e[2].elapsed_time(e[3]) for e in ev)
    att_mean = sum(e[2].elapsed_time(e[3]) for e in ev) / len(ev)
    ms_step = total_ms / args.steps
    status = abatt.read_status(ws_small) | abatt.read_status(ws_sel) | abatt.read_status(ws_att)

    c = counts.cpu().numpy().astype(np.int64)
    idx_h = idx.cpu().numpy()
    bpt = 128 // w.Bk
    # executed tiles: every row runs its own drawn blocks, 128/Bk per tile
    # (pairs of neighbouring rows share the gathers of common tiles, not the math)
    last = w.nK - 1
    tail = w.N - last * w.Bk
    keys = np.zeros(rows, dtype=np.int64)
    for r in range(rows):
        L = c[r]
        keys[r] = L * w.Bk - (w.Bk - tail if L and idx_h[r, :L][-1] == last else 0)
    tiles = int(((c + bpt - 1) // bpt).sum())
    exec_flop = tiles * 4.0 * 128 * 128 * w.d
    # algorithmic work: valid query rows x valid drawn keys
    nrows_q = np.minimum(128, w.N - (np.arange(rows) % w.nQ) * 128)
    alg_flop = float((4.0 * w.d * nrows_q * keys).sum())
    dense_flop = 4.0 * w.B * w.H * w.N * w.N * w.d
    skip = 1.0 - float((nrows_q * keys).sum()) / (w.B * w.H * w.N * float(w.N))

    pk, src = peaks()
    peak = float(pk.get("bf16_tflops_sustained") or pk["bf16_tflops"])
    achieved = alg_flop / (att_mean * 1e-3) / 1e12
    # blocks the two rows of a pair both drew (gathered once for both), over
    # the blocks either drew
    both = either = 0
    for r in range(0, rows - 1, 2):
        if (r % w.nQ) % 2 or r // w.nQ != (r + 1) // w.nQ:
            continue
        a0, a1 = idx_h[r, :c[r]], idx_h[r + 1, :c[r + 1]]
        k = np.intersect1d(a0, a1, assume_unique=True).size
        both += k
        either += a0.size + a1.size - k

    line = {
        "metric": METRIC,
        "value": job_value(dense_flop, world, ms_step),
        "unit": "TFLOPS (dense-equivalent)",
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "budget_bp": w.budget_bp, "kv_block": w.Bk, "clusters": w.clusters,
                   "kmeans_iters": w.iters, "selection": args.selection,
                   "scoring": args.scoring, "draws": args.draws,
                   "per_rank": "one batch element per GPU",
                   "l2": "inputs (Q,K,V 2.3 GB) exceed the 126 MB L2; no flush"},
        "stages_ms": {"select": sel_ms, "sample": smp_ms, "attention": att_ms},
        "attention_ms": att_ms,
        "selector_sampler_share": (sel_ms + smp_ms) / (sel_ms + smp_ms + att_ms),
        "realized_skip": skip,
        "pair_shared_fraction": both / max(either, 1),
        "executed_tflops_attention": exec_flop / (att_mean * 1e-3) / 1e12,
        "algorithmic_tflops_attention": achieved,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": attention_traffic(rows),
                     "kernel": "gather_attn_kernel", "flops": "algorithmic (valid query rows x drawn keys)",
                     "peak_source": f"{src} bf16 sustained"},
        "device_status": status,
        "gpu_launches": 7 * args.steps,
        "clocks": clk.summary(),
    }

    if not args.no_keep_all:
        line["keep_all"] = keep_all(abatt, cfg, Q, K, V, w, O, ws_att, stream)
    if not args.no_e2e:
        line["e2e"] = e2e(abatt, cfg, Qc, Kc, Vc, dev, w, args, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:  # the host baseline: one process alone
        line["cpu_baseline"] = cpu_baseline(w, Qc, Kc, Vc)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def keep_all(abatt, cfg, Q, K, V, w, O, ws, stream):
    """The same attention kernel fed every key block with weight 1 (dense
    attention through the gather path), timed the same way."""
    import torch

    rows, nK = w.rows, w.nK
    counts = torch.full((rows,), nK, dtype=torch.int32, device=Q.device)
    idx = torch.arange(nK, dtype=torch.int32, device=Q.device).repeat(rows, 1)
    logw = torch.zeros((rows, nK), dtype=torch.float32, device=Q.device)
    for _ in range(2):
        abatt.attention(Q, K, V, counts, idx, logw, cfg, out=O, workspace=ws, stream=stream)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    reps = 3
    a.record(stream)
    for _ in range(reps):
        abatt.attention(Q, K, V, counts, idx, logw, cfg, out=O, workspace=ws, stream=stream)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    dense = 4.0 * w.B * w.H * w.N * w.N * w.d
    tiles = rows * ((nK + 128 // w.Bk - 1) // (128 // w.Bk))
    return {"attention_ms": ms, "dense_tflops": dense / (ms * 1e-3) / 1e12,
            "executed_tflops": tiles * 4.0 * 128 * 128 * w.d / (ms * 1e-3) / 1e12}


def e2e(abatt, cfg, Qc, Kc, Vc, dev, w, args, world):
    """Same metric through the public host-to-host call: every step copies
    Q, K, V from pinned host memory to the device and O back, through
    abatt.HostPipeline (abatt_forward over chunks of heads, the copies of one
    chunk overlapped with the compute of the previous one)."""
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
    dense = 4.0 * w.B * w.H * w.N * w.N * w.d
    nbytes = Qc.numel() * 2
    return {"value": job_value(dense, world, ms), "unit": "TFLOPS (dense-equivalent)",
            "ms_per_step": ms, "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
            "steps": steps, "heads_per_chunk": pipe.hc, "device_status": pipe.status()}


if __name__ == "__main__":
    main()
