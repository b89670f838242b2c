"""C-ABI checks that need no GPU: the library loads, exports every entry
point declared in include/abatt.h, and rejects bad arguments on the host
before touching the device."""
import ctypes
import os
import re

import pytest

from block_sparse_attention_20_b200 import abatt, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return abatt.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "abatt.h")).read()
    return sorted(set(re.findall(r"^\S.*?\b(abatt_\w+)\(", src, flags=re.M)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 10
    assert sorted(abatt.EXPORTS) == names
    for n in names:
        assert hasattr(L, n), n


def test_version_and_status_strings(L):
    assert re.match(r"\d+\.\d+\.\d+$", abatt.version())
    for code in range(9):
        assert abatt.status_string(code) not in ("", "unknown status")
    assert abatt.status_string(99) == "unknown status"


def _ws(shape, cfg, call=abatt.CALL_FORWARD):
    return abatt.workspace_size(call, shape, cfg)


def test_workspace_sizes():
    cfg = abatt.Config(clusters=8, budget_bp=800)
    B, H, N, d = 1, 40, 75600, 128
    fwd = _ws((B, H, N, d), cfg)
    sel = _ws((B, H, N, d), cfg, abatt.CALL_SELECT)
    att = _ws((B, H, N, d), cfg, abatt.CALL_ATTENTION)
    assert _ws((B, H, N, d), cfg, abatt.CALL_SAMPLE) == 256
    rows, nK = 40 * 591, 4725
    pairs = 40 * 296  # neighbouring query blocks of a head, 591 per head
    # attention: per pair the union list (block, two log-weights) of at most nK blocks
    assert att >= 256 + pairs * nK * 12
    # forward holds the selector's and attention's scratch plus p and capacity-nK lists
    assert fwd >= sel + (att - 256) + rows * nK * 12 + rows * 4
    assert fwd < 8 * 2**30


@pytest.mark.parametrize("shape,kw,code", [
    ((1, 1, 100, 96), {}, 2),            # d not in {64, 128}
    ((1, 1, 100, 64), {"q_block": 64}, 2),
    ((1, 1, 100, 64), {"kv_block": 8}, 2),
    ((1, 1, 100, 64), {"clusters": 17}, 2),
    ((1, 1, 100, 64), {"clusters": 0}, 2),
    ((1, 1, 100, 64), {"kmeans_iters": 65}, 2),
    ((1, 1, 16 * 32768, 64), {}, 2),      # nK > 32767
    ((0, 1, 100, 64), {}, 1),
    ((1, 1, 0, 64), {}, 1),
    ((1, 1, 100, 64), {"budget_bp": -1}, 1),
    ((1, 1, 100, 64), {"scale": 0.0}, 1),
    ((1, 1, 100, 64), {"scale": float("nan")}, 1),
    ((1, 1, 100, 64), {"head_offset": -1}, 1),
    ((1, 1, 100, 64), {"batch_offset": -3}, 1),
    ((1, 1, 100, 64), {"selection": 2}, 1),
    ((1, 1, 100, 64), {"scoring": 3}, 1),
    ((1, 1, 100, 64), {"layout": 2}, 1),
    ((1, 1, 100, 64), {"draws": 2}, 1),
    ((1, 1, 16 * 10241, 64), {"selection": 1}, 2),   # top-M needs nK <= 10240
])
def test_validation(shape, kw, code):
    with pytest.raises(abatt.AbattError) as e:
        _ws(shape, abatt.Config(**kw))
    assert e.value.code == code


def test_host_side_rejections_before_any_device_call(L):
    sh = abatt._Shape(1, 2, 256, 64)
    cfg = abatt.Config()._c(64)
    P = ctypes.c_void_p
    # null tensors
    assert L.abatt_select(None, None, ctypes.byref(sh), ctypes.byref(cfg), None, None, None,
                          None, 0, None) == 1
    assert L.abatt_attention(None, None, None, ctypes.byref(sh), ctypes.byref(cfg), None, None,
                             None, 16, None, None, None, 0, None) == 1
    assert L.abatt_forward(None, None, None, ctypes.byref(sh), ctypes.byref(cfg), None, None,
                           None, 0, None) == 1
    # misaligned tensor pointers (never dereferenced)
    odd = P(0x1001)
    assert L.abatt_forward(odd, odd, odd, ctypes.byref(sh), ctypes.byref(cfg), odd, None,
                           P(0x100000), 1 << 30, None) == 3
    # missing / small / misaligned workspace
    ok = P(0x100000)
    assert L.abatt_forward(ok, ok, ok, ctypes.byref(sh), ctypes.byref(cfg), ok, None, None, 0,
                           None) == 4
    assert L.abatt_forward(ok, ok, ok, ctypes.byref(sh), ctypes.byref(cfg), ok, None, ok, 255,
                           None) == 4
    assert L.abatt_forward(ok, ok, ok, ctypes.byref(sh), ctypes.byref(cfg), ok, None,
                           P(0x100010), 1 << 30, None) == 3
    # sample: capacity must be positive
    assert L.abatt_sample(ok, ctypes.byref(sh), ctypes.byref(cfg), ok, ok, ok, 0, ok, 256,
                          None) == 1
    # null shape / config
    assert L.abatt_forward(ok, ok, ok, None, ctypes.byref(cfg), ok, None, ok, 1 << 30, None) == 1
    size = ctypes.c_size_t()
    assert L.abatt_workspace_size(7, ctypes.byref(sh), ctypes.byref(cfg), ctypes.byref(size)) == 1
    assert L.abatt_read_status(None, None, None) == 1


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(abatt, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(abatt, "_lib", None)
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        abatt.lib()


def test_config_struct_carries_the_slice_offsets():
    # abatt_config ends with batch_offset, head_offset after the 64-bit seed
    c = abatt.Config(seed=5, batch_offset=2, head_offset=7)._c(64)
    assert ctypes.sizeof(c) == 56
    assert (c.seed, c.batch_offset, c.head_offset) == (5, 2, 7)
    assert abatt._Config.selection.offset == 40 and abatt._Config.scoring.offset == 44
    assert abatt._Config.layout.offset == 48 and abatt._Config.draws.offset == 52
    assert abatt._Config.head_offset.offset == 36 and abatt._Config.batch_offset.offset == 32


def test_host_pipeline_streams_head_chunks_of_bhnd_only():
    # head chunks of a [B, N, H, d] tensor are not contiguous: refused before
    # any device allocation
    cfg = abatt.Config(layout=abatt.LAYOUT_BNHD)
    with pytest.raises(ValueError):
        abatt.HostPipeline((1, 4, 1024, 64), cfg)


def test_shape_of_follows_the_layout():
    import torch

    q = torch.empty((2, 300, 5, 64))
    sh = abatt._shape_of(q, abatt.Config(layout=abatt.LAYOUT_BNHD))
    assert (sh.B, sh.H, sh.N, sh.d) == (2, 5, 300, 64)
    sh = abatt._shape_of(q, abatt.Config())
    assert (sh.B, sh.H, sh.N, sh.d) == (2, 300, 5, 64)


def test_host_side_rejections_of_the_attention_launches_and_test_hooks(L):
    sh = abatt._Shape(1, 2, 256, 64)
    cfg = abatt.Config()._c(64)
    P = ctypes.c_void_p
    ok = P(0x100000)
    # plan: null lists, capacity < 1, missing workspace
    assert L.abatt_attention_plan(ctypes.byref(sh), ctypes.byref(cfg), None, ok, ok, 16, ok, 1 << 30,
                                  None) == 1
    assert L.abatt_attention_plan(ctypes.byref(sh), ctypes.byref(cfg), ok, ok, ok, 0, ok, 1 << 30,
                                  None) == 1
    assert L.abatt_attention_plan(ctypes.byref(sh), ctypes.byref(cfg), ok, ok, ok, 16, None, 0,
                                  None) == 4
    # planned: null and misaligned tensors, small workspace
    assert L.abatt_attention_planned(None, ok, ok, ctypes.byref(sh), ctypes.byref(cfg), ok, None, ok,
                                     1 << 30, None) == 1
    assert L.abatt_attention_planned(P(0x1001), ok, ok, ctypes.byref(sh), ctypes.byref(cfg), ok, None,
                                     ok, 1 << 30, None) == 3
    assert L.abatt_attention_planned(ok, ok, ok, ctypes.byref(sh), ctypes.byref(cfg), ok, None, ok, 255,
                                     None) == 4
    # test hooks: unknown hook, bad degree, negative size
    assert L.abatt_test_set(99, 0) == 1
    assert L.abatt_test_exp2_poly(ok, ok, 16, 5, None) == 1
    assert L.abatt_test_exp2_poly(None, ok, 16, 3, None) == 1
    assert L.abatt_test_exp2_poly(ok, ok, -1, 3, None) == 1
    # the no-alloc call: null inputs, then a shape beyond its scratch (before any device call)
    assert L.abatt_attention_noalloc(None, ok, ok, ctypes.byref(sh), ctypes.byref(cfg), ok, ok, ok, 16,
                                     ok, None, None, None) == 1
    big = abatt._Shape(1, 40, 75600, 128)
    assert L.abatt_attention_noalloc(ok, ok, ok, ctypes.byref(big), ctypes.byref(abatt.Config()._c(128)),
                                     ok, ok, ok, 16, ok, None, None, None) == 2


def test_binding_checks_buffer_shapes_dtypes_and_devices():
    import torch

    cpu = torch.device("cpu")
    rows, cap = 6, 10
    counts = torch.zeros(rows, dtype=torch.int32)
    idx = torch.zeros((rows, cap), dtype=torch.int32)
    logw = torch.zeros((rows, cap), dtype=torch.float32)
    assert abatt._check_lists(counts, idx, logw, rows, cpu) == cap
    with pytest.raises(ValueError, match="counts"):
        abatt._check_lists(counts[:5], idx, logw, rows, cpu)
    with pytest.raises(ValueError, match="idx"):
        abatt._check_lists(counts, idx.long(), logw, rows, cpu)
    with pytest.raises(ValueError, match="logw"):
        abatt._check_lists(counts, idx, logw[:, :9], rows, cpu)
    with pytest.raises(ValueError, match="capacity"):
        abatt._check_lists(counts, idx[:, :0], logw[:, :0], rows, cpu)
    with pytest.raises(ValueError, match="not contiguous"):
        abatt._check_lists(counts, idx, torch.zeros((cap, rows)).t(), rows, cpu)
    q = torch.zeros((1, 2, 300, 64), dtype=torch.bfloat16)
    sh = abatt._shape_of(q, abatt.Config())
    abatt._check_outputs(q, torch.zeros_like(q), torch.zeros((1, 2, 300)), sh)
    with pytest.raises(ValueError, match="out"):
        abatt._check_outputs(q, torch.zeros((1, 2, 299, 64), dtype=torch.bfloat16), None, sh)
    with pytest.raises(ValueError, match="out"):
        abatt._check_outputs(q, torch.zeros_like(q, dtype=torch.float32), None, sh)
    with pytest.raises(ValueError, match="lse"):
        abatt._check_outputs(q, None, torch.zeros((1, 2, 300), dtype=torch.float64), sh)
    # Q, K, V must be CUDA bf16 tensors of one shape
    with pytest.raises(ValueError):
        abatt._check_qkv(q, q, q)  # CPU tensors
