"""Host-side pieces of bench.py that need no GPU."""
import hashlib
import json
import os

import pytest

import bench
from block_sparse_attention_20_b200 import synth


def _key(tmp_path, sha):
    p = tmp_path / "key.json"
    p.write_text(json.dumps({"source_sha256_16": sha, "dram_bytes_per_query_block": 128577}))
    return str(p)


def _current_sha():
    csrc = os.path.join(bench.ROOT, "block_sparse_attention_20_b200", "csrc")
    return hashlib.sha256(bench.attention_source(csrc)).hexdigest()[:16]


def test_traffic_scales_with_query_blocks_for_the_profiled_kernel(tmp_path):
    key = _key(tmp_path, _current_sha())
    a = bench.attention_traffic(1000, key)
    b = bench.attention_traffic(3000, key)
    assert a == 128577 * 1000 and b == 3 * a


def test_traffic_is_withheld_for_another_kernel_source(tmp_path):
    assert bench.attention_traffic(1000, _key(tmp_path, "0" * 16)) is None
    assert bench.attention_traffic(1000, str(tmp_path / "missing.json")) is None


def test_committed_traffic_key_is_well_formed():
    if not os.path.exists(bench.TRAFFIC_KEY):
        pytest.skip("no committed counters")
    key = json.load(open(bench.TRAFFIC_KEY))
    assert len(key["source_sha256_16"]) == 16
    # the compulsory bytes of a query block: Q and O tiles plus its share of K, V
    assert 100_000 < key["dram_bytes_per_query_block"] < 140_000


def test_job_value_counts_every_rank():
    # 2e12 FLOP per rank on 4 ranks in 8 ms: 1,000 TFLOP/s for the whole job
    assert abs(bench.job_value(2e12, 4, 8.0) - 1000.0) < 1e-9


@pytest.mark.parametrize("H,world", [(40, 1), (40, 2), (40, 3), (40, 8), (24, 5), (2, 2)])
def test_head_split_covers_every_head_once(H, world):
    w = synth.WAN_14B.with_(H=H)
    seen = []
    for r in range(world):
        plan = bench.rank_plan(w, r, world, "heads")
        assert plan["batch_offset"] == 0 and plan["data_seed"] == w.seed and plan["philox_seed"] == w.seed
        assert plan["heads"] >= H // world
        seen += list(range(plan["head_offset"], plan["head_offset"] + plan["heads"]))
    assert seen == list(range(H))


def test_head_split_rejects_more_ranks_than_heads():
    with pytest.raises(ValueError):
        bench.rank_plan(synth.TINY, 0, 3, "heads")
    with pytest.raises(ValueError):
        bench.rank_plan(synth.TINY, 0, 1, "rows")


def test_both_arms_describe_the_workload_with_the_same_config():
    args = bench.parse([])
    cfg = bench.bench_config(synth.WAN_14B, args)
    assert cfg["workload"] == "wan14b-720p" and cfg["N"] == 75600 and cfg["kmeans_iters"] == 5
    assert {"selection", "scoring", "draws", "clusters", "budget_bp", "kv_block"} <= set(cfg)


def test_roofline_peaks_burst_and_clock_scaled():
    pk = {"bf16_tflops": 1653.2, "bf16_tflops_sustained": 1402.4,
          "clocks_under_load": {"sm_mhz_median": 1342.0}}
    burst, scaled = bench.roofline_peaks(pk, 1900.0)
    assert burst == 1653.2
    assert abs(scaled - 1402.4 * 1900.0 / 1342.0) < 1e-9
    assert bench.roofline_peaks({"bf16_tflops": 1.0}, 1900.0) == (1.0, None)
