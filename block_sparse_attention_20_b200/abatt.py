"""ctypes binding of the ``abatt`` C ABI (``include/abatt.h``).

Argument marshalling only: torch supplies device memory and the current
stream; every step of the path runs in ``libabatt.so``.  If the library is
missing this module raises -- there is no CPU fallback.

Names follow the abstract of "Accurate Block Attention (AB-Attention)":
``select`` (IBCS block probabilities), ``sample`` (SIP draw and
log-weights), ``attention`` (gather attention) and ``forward`` (all three).
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libabatt.so")

CALL_SELECT, CALL_SAMPLE, CALL_ATTENTION, CALL_FORWARD = 0, 1, 2, 3
DEVFLAG_CAPACITY, DEVFLAG_TIMEOUT, DEVFLAG_BADLIST = 0x1, 0x2, 0x4

# Every symbol declared in include/abatt.h.
EXPORTS = (
    "abatt_workspace_size", "abatt_select", "abatt_sample", "abatt_attention", "abatt_forward",
    "abatt_forward_intermediates", "abatt_read_status", "abatt_clear_status",
    "abatt_status_string", "abatt_version", "abatt_attention_noalloc",
)


class AbattError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} (status {code})")
        self.code = code


class _Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int)]


class _Config(ctypes.Structure):
    _fields_ = [("q_block", ctypes.c_int), ("kv_block", ctypes.c_int), ("clusters", ctypes.c_int),
                ("kmeans_iters", ctypes.c_int), ("budget_bp", ctypes.c_int),
                ("scale", ctypes.c_float), ("seed", ctypes.c_uint64)]


@dataclass(frozen=True)
class Config:
    """Method parameters (see abatt_config in include/abatt.h)."""

    q_block: int = 128
    kv_block: int = 16
    clusters: int = 8
    kmeans_iters: int = 5
    budget_bp: int = 1000
    scale: float | None = None  # default 1/sqrt(d)
    seed: int = 0

    def _c(self, d: int) -> _Config:
        s = self.scale if self.scale is not None else 1.0 / math.sqrt(d)
        return _Config(self.q_block, self.kv_block, self.clusters, self.kmeans_iters,
                       self.budget_bp, s, self.seed & (2**64 - 1))


_lock = threading.Lock()
_lib = None


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m block_sparse_attention_20_b200.build`"
                " (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        P, S, i32, sz = ctypes.c_void_p, ctypes.POINTER(_Shape), ctypes.c_int, ctypes.c_size_t
        C = ctypes.POINTER(_Config)
        L.abatt_workspace_size.argtypes = [i32, S, C, ctypes.POINTER(sz)]
        L.abatt_select.argtypes = [P, P, S, C, P, P, P, P, sz, P]
        L.abatt_sample.argtypes = [P, S, C, P, P, P, i32, P, sz, P]
        L.abatt_attention.argtypes = [P, P, P, S, C, P, P, P, i32, P, P, P, sz, P]
        L.abatt_forward.argtypes = [P, P, P, S, C, P, P, P, sz, P]
        L.abatt_attention_noalloc.argtypes = [P, P, P, S, C, P, P, P, i32, P, P, P, P]
        L.abatt_forward_intermediates.argtypes = [P, S, C, ctypes.POINTER(P), ctypes.POINTER(P),
                                                  ctypes.POINTER(P), ctypes.POINTER(P)]
        L.abatt_read_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32), P]
        L.abatt_clear_status.argtypes = [P, P]
        L.abatt_status_string.argtypes = [i32]
        L.abatt_status_string.restype = ctypes.c_char_p
        L.abatt_version.restype = ctypes.c_char_p
        for name in EXPORTS:
            if name not in ("abatt_status_string", "abatt_version"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
        return L


def status_string(code: int) -> str:
    return lib().abatt_status_string(int(code)).decode()


def version() -> str:
    return lib().abatt_version().decode()


def _check(code: int, what: str):
    if code != 0:
        raise AbattError(code, what)


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _shape_of(q) -> _Shape:
    B, H, N, d = q.shape
    return _Shape(B, H, N, d)


def _geom(shape: _Shape, cfg: Config):
    nQ = -(-shape.N // cfg.q_block)
    nK = -(-shape.N // cfg.kv_block)
    return nQ, nK, shape.B * shape.H * nQ


def _check_bf16(*ts):
    import torch
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("Q, K, V must be contiguous CUDA bfloat16 tensors [B, H, N, d]")


def workspace_size(call: int, shape, cfg: Config) -> int:
    sh = shape if isinstance(shape, _Shape) else _Shape(*shape)
    out = ctypes.c_size_t()
    _check(lib().abatt_workspace_size(call, ctypes.byref(sh), ctypes.byref(cfg._c(sh.d)),
                                      ctypes.byref(out)), "abatt_workspace_size")
    return out.value


def _workspace(call, sh, cfg, device, workspace):
    import torch
    need = workspace_size(call, sh, cfg)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    elif workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace too small: {need} bytes needed")
    return workspace


def select(q, k, cfg: Config, *, p=None, want_centroids=False, workspace=None, stream=None):
    """IBCS block probabilities p [B*H*nQ, nK] (fp32).

    With ``want_centroids`` also returns the fp32 centroids [rows, C, d] and
    cluster sizes [rows, C]."""
    import torch
    _check_bf16(q, k)
    sh = _shape_of(q)
    nQ, nK, rows = _geom(sh, cfg)
    if p is None:
        p = torch.empty((rows, nK), dtype=torch.float32, device=q.device)
    cent = sizes = None
    if want_centroids:
        cent = torch.empty((rows, cfg.clusters, sh.d), dtype=torch.float32, device=q.device)
        sizes = torch.empty((rows, cfg.clusters), dtype=torch.int32, device=q.device)
    ws = _workspace(CALL_SELECT, sh, cfg, q.device, workspace)
    _check(lib().abatt_select(_ptr(q), _ptr(k), ctypes.byref(sh), ctypes.byref(cfg._c(sh.d)),
                              _ptr(p), _ptr(cent), _ptr(sizes), _ptr(ws), ws.numel(),
                              _stream(stream)), "abatt_select")
    return (p, cent, sizes) if want_centroids else p


def sample(p, shape, cfg: Config, *, capacity=None, out=None, workspace=None, stream=None):
    """SIP draw: returns (counts [rows], idx [rows, cap], logw [rows, cap], workspace)."""
    import torch
    sh = shape if isinstance(shape, _Shape) else _Shape(*shape)
    nQ, nK, rows = _geom(sh, cfg)
    if p.dtype != torch.float32 or not p.is_cuda or p.shape != (rows, nK) or not p.is_contiguous():
        raise ValueError(f"p must be a contiguous CUDA float32 tensor of shape {(rows, nK)}")
    cap = nK if capacity is None else int(capacity)
    if out is None:
        counts = torch.empty(rows, dtype=torch.int32, device=p.device)
        idx = torch.empty((rows, cap), dtype=torch.int32, device=p.device)
        logw = torch.empty((rows, cap), dtype=torch.float32, device=p.device)
    else:
        counts, idx, logw = out
    ws = _workspace(CALL_SAMPLE, sh, cfg, p.device, workspace)
    _check(lib().abatt_sample(_ptr(p), ctypes.byref(sh), ctypes.byref(cfg._c(sh.d)), _ptr(counts),
                              _ptr(idx), _ptr(logw), cap, _ptr(ws), ws.numel(), _stream(stream)),
           "abatt_sample")
    return counts, idx, logw, ws


def attention(q, k, v, counts, idx, logw, cfg: Config, *, out=None, want_lse=False,
              workspace=None, stream=None):
    """Gather attention over the listed blocks.  Returns O (and lse)."""
    import torch
    _check_bf16(q, k, v)
    sh = _shape_of(q)
    cap = idx.shape[1]
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((sh.B, sh.H, sh.N), dtype=torch.float32, device=q.device) if want_lse else None
    ws = _workspace(CALL_ATTENTION, sh, cfg, q.device, workspace)
    _check(lib().abatt_attention(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(sh),
                                 ctypes.byref(cfg._c(sh.d)), _ptr(counts), _ptr(idx), _ptr(logw),
                                 cap, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "abatt_attention")
    return (out, lse) if want_lse else out


NOALLOC_SCRATCH_BYTES = 64 << 20


def attention_noalloc(q, k, v, counts, idx, logw, cfg: Config, *, out, lse=None, dev_status=None,
                      stream=None):
    """Gather attention through the entry point that allocates nothing.

    For callers that cannot allocate device memory: its scratch is a fixed
    64 MiB array inside the library, shared by every call on a device (calls
    that overlap on the GPU race on it).  The caller supplies every input and
    output buffer, including `out` (and `lse`, `dev_status` if wanted)."""
    _check_bf16(q, k, v)
    sh = _shape_of(q)
    _check(lib().abatt_attention_noalloc(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(sh),
                                         ctypes.byref(cfg._c(sh.d)), _ptr(counts), _ptr(idx),
                                         _ptr(logw), idx.shape[1], _ptr(out), _ptr(lse),
                                         _ptr(dev_status), _stream(stream)),
           "abatt_attention_noalloc")
    return out


def forward(q, k, v, cfg: Config, *, out=None, want_lse=False, workspace=None, stream=None):
    """The whole path.  Returns O (and lse); pass ``workspace`` to keep the
    intermediates (see :func:`intermediates`)."""
    import torch
    _check_bf16(q, k, v)
    sh = _shape_of(q)
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((sh.B, sh.H, sh.N), dtype=torch.float32, device=q.device) if want_lse else None
    ws = _workspace(CALL_FORWARD, sh, cfg, q.device, workspace)
    _check(lib().abatt_forward(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(sh),
                               ctypes.byref(cfg._c(sh.d)), _ptr(out), _ptr(lse), _ptr(ws),
                               ws.numel(), _stream(stream)), "abatt_forward")
    return (out, lse) if want_lse else out


def intermediates(workspace, shape, cfg: Config):
    """Views (p, counts, idx, logw) into a FORWARD workspace."""
    import torch
    sh = shape if isinstance(shape, _Shape) else _Shape(*shape)
    nQ, nK, rows = _geom(sh, cfg)
    ptrs = [ctypes.c_void_p() for _ in range(4)]
    _check(lib().abatt_forward_intermediates(_ptr(workspace), ctypes.byref(sh),
                                             ctypes.byref(cfg._c(sh.d)),
                                             *[ctypes.byref(x) for x in ptrs]),
           "abatt_forward_intermediates")
    base = workspace.data_ptr()

    def view(ptr, n, dtype):
        off = ptr.value - base
        return workspace[off:off + n * torch.tensor([], dtype=dtype).element_size()].view(dtype)

    p = view(ptrs[0], rows * nK, torch.float32).view(rows, nK)
    counts = view(ptrs[1], rows, torch.int32)
    idx = view(ptrs[2], rows * nK, torch.int32).view(rows, nK)
    logw = view(ptrs[3], rows * nK, torch.float32).view(rows, nK)
    return p, counts, idx, logw


def read_status(workspace, stream=None) -> int:
    """Device status bits of a workspace (synchronises the stream)."""
    flags = ctypes.c_uint32()
    code = lib().abatt_read_status(_ptr(workspace), ctypes.byref(flags), _stream(stream))
    if code not in (0, 8):
        _check(code, "abatt_read_status")
    return flags.value
