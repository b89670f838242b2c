"""Host-side pieces of bench.py that need no GPU."""
import bench


def test_traffic_scales_with_query_blocks_for_the_profiled_kernel():
    a = bench.attention_traffic(1000)
    b = bench.attention_traffic(3000)
    assert a is not None and a > 0 and b == 3 * a
    # the compulsory bytes of a query block: Q and O tiles plus its share of K, V
    assert 100_000 < a / 1000 < 140_000


def test_traffic_is_withheld_for_another_kernel_source(monkeypatch):
    real = bench.attention_source
    monkeypatch.setattr(bench, "attention_source", lambda csrc: real(csrc) + b" changed")
    assert bench.attention_traffic(1000) is None


def test_job_value_counts_every_rank():
    # 2e12 FLOP per rank on 4 ranks in 8 ms: 1,000 TFLOP/s for the whole job
    assert abs(bench.job_value(2e12, 4, 8.0) - 1000.0) < 1e-9
