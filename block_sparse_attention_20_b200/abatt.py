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
SELECT_SIP, SELECT_TOPK = 0, 1
SCORE_KEYS, SCORE_BLOCK_MEANS = 0, 1
LAYOUT_BHND, LAYOUT_BNHD = 0, 1
DRAWS_INDEPENDENT, DRAWS_PAIRED = 0, 1
DEVFLAG_CAPACITY, DEVFLAG_TIMEOUT, DEVFLAG_BADLIST = 0x1, 0x2, 0x4
NOALLOC_STATUS_PENDING = 0xFFFFFFFF
TEST_WAIT_NS, TEST_STALL = 1, 2
TEST_STALL_ATTENTION, TEST_STALL_SCORE = 0x1, 0x2

# Every symbol declared in include/abatt.h.
EXPORTS = (
    "abatt_workspace_size", "abatt_select", "abatt_sample", "abatt_attention", "abatt_forward",
    "abatt_forward_intermediates", "abatt_read_status", "abatt_clear_status",
    "abatt_status_string", "abatt_version", "abatt_attention_noalloc",
    "abatt_attention_plan", "abatt_attention_planned", "abatt_test_set", "abatt_test_exp2_poly",
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
                ("scale", ctypes.c_float), ("seed", ctypes.c_uint64),
                ("batch_offset", ctypes.c_int), ("head_offset", ctypes.c_int),
                ("selection", ctypes.c_int), ("scoring", ctypes.c_int),
                ("layout", ctypes.c_int), ("draws", ctypes.c_int)]


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
    batch_offset: int = 0  # global index of the call's first batch element
    head_offset: int = 0   # global index of the call's first head
    selection: int = 0     # SELECT_SIP (the method) or SELECT_TOPK (truncating baseline)
    scoring: int = 0       # SCORE_KEYS (the method as read) or SCORE_BLOCK_MEANS (coarse baseline)
    layout: int = 0        # LAYOUT_BHND ([B,H,N,d]) or LAYOUT_BNHD ([B,N,H,d])
    draws: int = 0         # DRAWS_INDEPENDENT or DRAWS_PAIRED (query blocks 2j, 2j+1 share uniforms)

    def _c(self, d: int) -> _Config:
        s = self.scale if self.scale is not None else 1.0 / math.sqrt(d)
        return _Config(self.q_block, self.kv_block, self.clusters, self.kmeans_iters,
                       self.budget_bp, s, self.seed & (2**64 - 1), self.batch_offset, self.head_offset,
                       self.selection, self.scoring, self.layout, self.draws)


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
        L.abatt_attention_plan.argtypes = [S, C, P, P, P, i32, P, sz, P]
        L.abatt_attention_planned.argtypes = [P, P, P, S, C, P, P, P, sz, P]
        L.abatt_test_set.argtypes = [i32, ctypes.c_uint64]
        L.abatt_test_exp2_poly.argtypes = [P, P, ctypes.c_int64, i32, P]
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


def _shape_of(q, cfg=None) -> _Shape:
    """(B, H, N, d) of a Q/K/V tensor in the layout cfg names."""
    if cfg is not None and cfg.layout == LAYOUT_BNHD:
        B, N, H, d = q.shape
    else:
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
            raise ValueError("Q, K, V must be contiguous CUDA bfloat16 tensors ([B, H, N, d], or "
                             "[B, N, H, d] with layout=LAYOUT_BNHD)")


def _check_qkv(q, k, v=None):
    """Q, K (and V): contiguous CUDA bf16 4-D tensors of one shape on one device."""
    ts = (q, k) if v is None else (q, k, v)
    _check_bf16(*ts)
    if q.dim() != 4:
        raise ValueError(f"Q must be 4-D, got shape {tuple(q.shape)}")
    for name, t in zip("KV", ts[1:]):
        if t.shape != q.shape or t.device != q.device:
            raise ValueError(f"{name} must have Q's shape {tuple(q.shape)} and device {q.device}, "
                             f"got {tuple(t.shape)} on {t.device}")


def _check_tensor(t, name, dtype, shape, device):
    import torch
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a torch tensor")
    if t.dtype != dtype or t.device != device or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)} on {device}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}"
                         f"{'' if t.is_contiguous() else ' (not contiguous)'}")


def _check_lists(counts, idx, logw, rows, device):
    """counts int32 [rows]; idx int32 and logw fp32 [rows, capacity] (capacity >= 1)."""
    import torch
    if idx.dim() != 2 or idx.shape[1] < 1:
        raise ValueError(f"idx must be [rows, capacity] with capacity >= 1, got {tuple(idx.shape)}")
    cap = idx.shape[1]
    _check_tensor(counts, "counts", torch.int32, (rows,), device)
    _check_tensor(idx, "idx", torch.int32, (rows, cap), device)
    _check_tensor(logw, "logw", torch.float32, (rows, cap), device)
    return cap


def _check_outputs(q, out, lse, sh):
    import torch
    if out is not None:
        _check_tensor(out, "out", torch.bfloat16, q.shape, q.device)
    if lse is not None:
        _check_tensor(lse, "lse", torch.float32, (sh.B, sh.H, sh.N), q.device)


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
    _check_qkv(q, k)
    sh = _shape_of(q, cfg)
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
    _check_qkv(q, k, v)
    sh = _shape_of(q, cfg)
    cap = _check_lists(counts, idx, logw, _geom(sh, cfg)[2], q.device)
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((sh.B, sh.H, sh.N), dtype=torch.float32, device=q.device) if want_lse else None
    _check_outputs(q, out, lse, sh)
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
    output buffer, including `out` (and `lse`, `dev_status` if wanted); this
    wrapper checks their shapes, dtypes and devices and allocates nothing."""
    import torch
    _check_qkv(q, k, v)
    sh = _shape_of(q, cfg)
    cap = _check_lists(counts, idx, logw, _geom(sh, cfg)[2], q.device)
    if out is None:
        raise ValueError("out is required (the call allocates nothing)")
    _check_outputs(q, out, lse, sh)
    if dev_status is not None:
        if dev_status.dtype not in (torch.int32, torch.uint32) or dev_status.numel() != 1 \
                or dev_status.device != q.device:
            raise ValueError("dev_status must be a one-element int32 or uint32 tensor on Q's device")
    _check(lib().abatt_attention_noalloc(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(sh),
                                         ctypes.byref(cfg._c(sh.d)), _ptr(counts), _ptr(idx),
                                         _ptr(logw), cap, _ptr(out), _ptr(lse),
                                         _ptr(dev_status), _stream(stream)),
           "abatt_attention_noalloc")
    return out


def attention_plan(shape, counts, idx, logw, cfg: Config, *, workspace, stream=None):
    """First launch of :func:`attention`: the pair segments, into `workspace`
    (an ATTENTION workspace; its status word is cleared)."""
    sh = shape if isinstance(shape, _Shape) else _Shape(*shape)
    cap = _check_lists(counts, idx, logw, _geom(sh, cfg)[2], counts.device)
    ws = _workspace(CALL_ATTENTION, sh, cfg, counts.device, workspace)
    _check(lib().abatt_attention_plan(ctypes.byref(sh), ctypes.byref(cfg._c(sh.d)), _ptr(counts), _ptr(idx),
                                      _ptr(logw), cap, _ptr(ws), ws.numel(), _stream(stream)),
           "abatt_attention_plan")
    return ws


def attention_planned(q, k, v, cfg: Config, *, workspace, out=None, want_lse=False, stream=None):
    """Second launch of :func:`attention`: the gather-attention kernel on the
    plan that :func:`attention_plan` left in `workspace`."""
    import torch
    _check_qkv(q, k, v)
    sh = _shape_of(q, cfg)
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((sh.B, sh.H, sh.N), dtype=torch.float32, device=q.device) if want_lse else None
    _check_outputs(q, out, lse, sh)
    ws = _workspace(CALL_ATTENTION, sh, cfg, q.device, workspace)
    _check(lib().abatt_attention_planned(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(sh),
                                         ctypes.byref(cfg._c(sh.d)), _ptr(out), _ptr(lse), _ptr(ws),
                                         ws.numel(), _stream(stream)), "abatt_attention_planned")
    return (out, lse) if want_lse else out


def test_set(hook: int, value: int) -> None:
    """Test hook of the library (TEST_WAIT_NS, TEST_STALL; see abatt_test_set)."""
    _check(lib().abatt_test_set(int(hook), int(value) & (2**64 - 1)), "abatt_test_set")


def test_exp2_poly(x, degree: int, stream=None):
    """2^x (fp32 CUDA tensor) through the kernels' FMA-pipe polynomial."""
    import torch
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA float32 tensor")
    y = torch.empty_like(x)
    _check(lib().abatt_test_exp2_poly(_ptr(x), _ptr(y), x.numel(), int(degree), _stream(stream)),
           "abatt_test_exp2_poly")
    return y


def forward(q, k, v, cfg: Config, *, out=None, want_lse=False, workspace=None, stream=None):
    """The whole path.  Returns O (and lse); pass ``workspace`` to keep the
    intermediates (see :func:`intermediates`)."""
    import torch
    _check_qkv(q, k, v)
    sh = _shape_of(q, cfg)
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((sh.B, sh.H, sh.N), dtype=torch.float32, device=q.device) if want_lse else None
    _check_outputs(q, out, lse, sh)
    ws = _workspace(CALL_FORWARD, sh, cfg, q.device, workspace)
    _check(lib().abatt_forward(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(sh),
                               ctypes.byref(cfg._c(sh.d)), _ptr(out), _ptr(lse), _ptr(ws),
                               ws.numel(), _stream(stream)), "abatt_forward")
    return (out, lse) if want_lse else out


class HostPipeline:
    """The whole path on pinned host tensors, with the copies overlapped.

    Heads are independent and the sampler draws with global head indices
    (``Config.head_offset``), so the problem is split into chunks of
    ``heads_per_chunk`` heads of one batch element; while chunk j runs
    ``abatt_forward`` on the compute stream, chunk j+1's Q, K, V travel
    host -> device on a copy stream and chunk j-1's O travels back on a third.
    The result equals one ``forward`` over the whole problem.  Device buffers
    (two chunk sets) and one FORWARD workspace per chunk are allocated once,
    here; every chunk's status word stays readable (:meth:`status`).
    """

    def __init__(self, shape, cfg: Config, *, heads_per_chunk: int = 5, device=None):
        import torch
        if cfg.layout != LAYOUT_BHND:
            raise ValueError("HostPipeline streams head chunks of [B, H, N, d] tensors (layout=LAYOUT_BHND)")
        self.B, self.H, self.N, self.d = shape
        self.cfg = cfg
        self.hc = max(1, min(heads_per_chunk, self.H))
        self.dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        self.chunks = [(b, h0, min(h0 + self.hc, self.H)) for b in range(self.B)
                       for h0 in range(0, self.H, self.hc)]
        cshape = (1, self.hc, self.N, self.d)
        self.buf = [[torch.empty(cshape, dtype=torch.bfloat16, device=self.dev) for _ in range(4)]
                    for _ in range(2)]  # (Q, K, V, O) x 2
        self.ws = [torch.empty(workspace_size(CALL_FORWARD, (1, h1 - h0, self.N, self.d), cfg),
                               dtype=torch.uint8, device=self.dev) for _, h0, h1 in self.chunks]
        self.s_in, self.s_comp, self.s_out = (torch.cuda.Stream(self.dev) for _ in range(3))

    def __call__(self, q, k, v, out):
        """q, k, v, out: pinned host bf16 [B, H, N, d].  Enqueues everything;
        the current stream waits for the last copy of O."""
        import torch
        n = len(self.chunks)
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_comp = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        self.s_in.wait_stream(torch.cuda.current_stream(self.dev))
        for j, (b, h0, h1) in enumerate(self.chunks):
            Qd, Kd, Vd, Od = (t[:, :h1 - h0] for t in self.buf[j % 2])
            with torch.cuda.stream(self.s_in):
                if j >= 2:
                    self.s_in.wait_event(ev_out[j - 2])  # buffer set free again
                Qd.copy_(q[b:b + 1, h0:h1], non_blocking=True)
                Kd.copy_(k[b:b + 1, h0:h1], non_blocking=True)
                Vd.copy_(v[b:b + 1, h0:h1], non_blocking=True)
                ev_in[j].record(self.s_in)
            self.s_comp.wait_event(ev_in[j])
            c = Config(**{**self.cfg.__dict__, "batch_offset": self.cfg.batch_offset + b,
                          "head_offset": self.cfg.head_offset + h0})
            forward(Qd, Kd, Vd, c, out=Od, workspace=self.ws[j], stream=self.s_comp)
            ev_comp[j].record(self.s_comp)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(ev_comp[j])
                out[b:b + 1, h0:h1].copy_(Od, non_blocking=True)
                ev_out[j].record(self.s_out)
        torch.cuda.current_stream(self.dev).wait_event(ev_out[n - 1])
        for e in ev_out[:-1]:
            torch.cuda.current_stream(self.dev).wait_event(e)
        return out

    def status(self) -> int:
        """OR of every chunk's device status word (synchronises)."""
        f = 0
        for w in self.ws:
            f |= read_status(w)
        return f


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
