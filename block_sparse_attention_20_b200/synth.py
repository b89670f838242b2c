"""Seeded synthetic video-token inputs (prototype-Voronoi Q/K/V).

This module is shared by the tests, the benchmark and the oracle checks.  It
holds no arithmetic of the attention method itself: it only draws inputs.

Stand-in for the activations of the video diffusion transformers the
AB-Attention abstract evaluates on (Wan2.1, HunyuanVideo), whose weights are
not available.  Tokens sit on a latent (t, y, x) grid in raster order.  Each
head has P prototype vectors attached to P random seed points of the
normalised grid; a token takes the prototype of its nearest seed (ties to the
smallest seed index), so semantically similar tokens form spatio-temporal
Voronoi cells, the structure block-sparse video attention exploits.

Per head, in this draw order (numpy PCG64, one generator for the whole
tensor, heads in (beta, h) order):
  1. seeds ~ U[0,1]^3                  (P x 3, float64)
  2. prototypes ~ N(0, I_d)            (P x d, float64)
  3. Q = proto + noise * N(0,1)
  4. K = proto * (1 + 0.1 N(0,1)) + noise * N(0,1)
  5. V ~ N(0,1)
Noise draws (3-5) are float32 normals.  Values are cast to bf16, layout
[B, H, N, d].
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    """One synthetic workload.  Field names follow the abstract's notation."""

    name: str
    B: int
    H: int
    d: int
    grid: tuple  # latent (T, Hgrid, Wgrid); tokens = first N of the raster
    N: int
    prototypes: int
    clusters: int  # C, k-means clusters per query block
    budget_bp: int  # expected drawn blocks, basis points of nK
    Bq: int = 128
    Bk: int = 16
    iters: int = 5  # k-means rounds
    noise: float = 0.5
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def nQ(self) -> int:
        return -(-self.N // self.Bq)

    @property
    def nK(self) -> int:
        return -(-self.N // self.Bk)

    @property
    def shape(self) -> tuple:
        return (self.B, self.H, self.N, self.d)

    @property
    def rows(self) -> int:
        return self.B * self.H * self.nQ

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


def _grid_workload(name, B, H, d, grid, P, C, budget_bp, **kw) -> Workload:
    T, Hg, Wg = grid
    return Workload(name=name, B=B, H=H, d=d, grid=grid, N=T * Hg * Wg, prototypes=P,
                    clusters=C, budget_bp=budget_bp, **kw)


# The five workloads (sizes of the Wan2.1 / HunyuanVideo latent grids).
TINY = _grid_workload("tiny", 1, 2, 64, (4, 32, 32), 16, 4, 1000)
WAN_1_3B = _grid_workload("wan1.3b", 1, 12, 128, (21, 30, 52), 64, 8, 1000)
WAN_14B = _grid_workload("wan14b-720p", 1, 40, 128, (21, 45, 80), 128, 8, 800)
HUNYUAN = _grid_workload("hunyuanvideo", 1, 24, 128, (33, 45, 80), 128, 8, 1100)

WORKLOADS = {w.name: w for w in (TINY, WAN_1_3B, WAN_14B, HUNYUAN)}


def sweep(N: int, budget_pct: int, Bk: int) -> Workload:
    """Sweep point: H=24, d=128, T x 45 x 80 grid truncated to N tokens."""
    T = -(-N // 3600)
    return Workload(name=f"sweep-N{N}-b{budget_pct}-k{Bk}", B=1, H=24, d=128, grid=(T, 45, 80),
                    N=N, prototypes=128, clusters=8, budget_bp=100 * budget_pct, Bk=Bk)


SWEEP_N = (8192, 32768, 65536, 131072)
SWEEP_BUDGET = (5, 10, 25, 50, 100)
SWEEP_BK = (16, 32, 64, 128)


def token_coords(grid, N: int) -> np.ndarray:
    """Normalised (t, y, x) of the first N raster tokens, [N, 3] float64."""
    T, Hg, Wg = grid
    n = np.arange(N, dtype=np.int64)
    t = n // (Hg * Wg)
    y = (n // Wg) % Hg
    x = n % Wg

    def norm(v, size):
        return v.astype(np.float64) / (size - 1) if size > 1 else np.zeros(len(v))

    return np.stack([norm(t, T), norm(y, Hg), norm(x, Wg)], axis=1)


def nearest_seed(coords: np.ndarray, seeds: np.ndarray) -> np.ndarray:
    """Index of the nearest seed point per token; ties go to the smallest index."""
    best = np.zeros(len(coords), dtype=np.int64)
    bestd = np.full(len(coords), np.inf)
    for j in range(len(seeds)):
        dj = ((coords - seeds[j]) ** 2).sum(axis=1)
        better = dj < bestd
        best[better] = j
        bestd[better] = dj[better]
    return best


def generate(w: Workload, heads=None):
    """Draw Q, K, V for workload `w` as CPU torch bf16 tensors [B, H, N, d].

    `heads` (optional) restricts generation to the first `heads` heads of
    batch 0 -- the draw order makes these identical to the full tensor's."""
    import torch

    B, H, N, d, P = w.B, w.H, w.N, w.d, w.prototypes
    nh = B * H if heads is None else int(heads)
    rng = np.random.Generator(np.random.PCG64(w.seed))
    coords = token_coords(w.grid, N)
    out = [torch.empty((nh, N, d), dtype=torch.bfloat16) for _ in range(3)]
    for k in range(nh):
        seeds = rng.random((P, 3))
        proto = rng.standard_normal((P, d)).astype(np.float32)
        pt = proto[nearest_seed(coords, seeds)]
        q = pt + np.float32(w.noise) * rng.standard_normal((N, d), dtype=np.float32)
        kk = pt * (np.float32(1.0) + np.float32(0.1) * rng.standard_normal((N, d), dtype=np.float32))
        kk += np.float32(w.noise) * rng.standard_normal((N, d), dtype=np.float32)
        v = rng.standard_normal((N, d), dtype=np.float32)
        for dst, src in zip(out, (q, kk, v)):
            dst[k].copy_(torch.from_numpy(src).to(torch.bfloat16))
    if heads is None:
        return tuple(x.view(B, H, N, d) for x in out)
    return tuple(x.view(1, nh, N, d) for x in out)


def generate_on_device(w: Workload, device):
    """The same prototype-Voronoi recipe as `generate`, drawn on the GPU with
    torch's Philox generator (one stream per head, seeded from w.seed and the
    head), for workloads too large to draw on the host in reasonable time.
    Same distribution as `generate`, different numbers.  Returns [B, H, N, d]
    bf16 device tensors."""
    import torch

    B, H, N, d, P = w.B, w.H, w.N, w.d, w.prototypes
    coords = torch.from_numpy(token_coords(w.grid, N)).to(device=device, dtype=torch.float64)
    out = [torch.empty((B * H, N, d), dtype=torch.bfloat16, device=device) for _ in range(3)]
    for k in range(B * H):
        g = torch.Generator(device=device)
        g.manual_seed(int(w.seed) * 1000003 + k)
        seeds = torch.rand((P, 3), generator=g, device=device, dtype=torch.float64)
        proto = torch.randn((P, d), generator=g, device=device)
        # nearest seed, ties to the smallest index (argmin returns the first)
        near = torch.cdist(coords, seeds).argmin(dim=1)
        pt = proto[near]
        noise = float(w.noise)
        q = pt + noise * torch.randn((N, d), generator=g, device=device)
        kk = pt * (1.0 + 0.1 * torch.randn((N, d), generator=g, device=device))
        kk += noise * torch.randn((N, d), generator=g, device=device)
        v = torch.randn((N, d), generator=g, device=device)
        for dst, src in zip(out, (q, kk, v)):
            dst[k].copy_(src.to(torch.bfloat16))
    return tuple(x.view(B, H, N, d) for x in out)


def random_bf16(shape, seed: int, scale: float = 1.0):
    """Plain N(0, scale^2) bf16 tensor (for edge-case tests)."""
    import torch

    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal(shape, dtype=np.float32) * np.float32(scale)
    return torch.from_numpy(x).to(torch.bfloat16)


def random_probs(rows: int, nK: int, seed: int, concentration: float = 0.3) -> np.ndarray:
    """Per-row fp32 probability vectors with a heavy-tailed spread (Dirichlet
    draws), for sampler tests that do not need the selector."""
    rng = np.random.Generator(np.random.PCG64(seed))
    p = rng.dirichlet(np.full(nK, concentration), size=rows)
    return p.astype(np.float32)
