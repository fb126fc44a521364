"""Seeded synthetic inputs for block-sparse video attention.

This module is the only code shared by the CPU oracle and the CUDA path. It draws the
inputs of one attention call of a video diffusion transformer and nothing else: it holds
none of the method's arithmetic (no tiling, pooling, scoring, selection or attention).

The video DiT pages (HetA-DiT abstract; Token Radius Attention summary; VORTA summary)
describe Q, K, V of a spatio-temporal token grid whose attention is dominated by local
structure, with a few globally attended tokens. With no model weights available, the
tensors are a random linear projection of low-frequency sinusoids of the normalised
(t, y, x) coordinates, plus Gaussian noise, with a few "sink" tokens whose q, k, v rows are
scaled up. Token order is raster: n = (t*Hs + y)*Ws + x, layout [B, N, H, d].

Generator G(seed), with rng = numpy.random.default_rng(seed) (PCG64):
  1. phases phi ~ U(0, 2*pi), shape [3 axes, 3 frequencies] (axis order t, y, x);
  2. features (19 per token): for each axis a and f in {1, 2, 3}, sin(2*pi*f*u_a + phi)
     and cos(2*pi*f*u_a + phi) with u_t = t/T, u_y = y/Hs, u_x = x/Ws; then a constant 1;
  3. projections W_q, W_k, W_v ~ N(0, 1)/sqrt(19), each [H, 19, d], drawn in order q, k, v;
  4. X = features @ W_h + noise_std * eps, eps ~ N(0, 1) float32 of shape [B, N, H, d],
     drawn in order q, k, v;
  5. sink tokens: round(s*N) positions drawn without replacement; their rows of q, k and v
     (all heads, all batch items) are multiplied by 3;
  6. cast to bfloat16 (round to nearest even);
  7. difficulty: default_rng(seed + 100).random((B, NQT)) as float32, one value per
     (batch item, query tile), the stand-in for a learned per-region difficulty estimate.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

TILE_EDGE = 4
TILE_TOKENS = TILE_EDGE ** 3


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention call: geometry, generator settings and mask-rule settings."""

    name: str
    B: int
    H: int
    d: int
    T: int
    Hs: int
    Ws: int
    seed: int
    sink_frac: float = 0.01
    noise_std: float = 0.5
    # mask rule
    window_kind: int = 0          # 0: cube (Chebyshev) window, 1: window with temporal decay
    radius: int = 1
    topk: int = 0
    dense_fraction: float = 0.0   # rho: share of query tiles routed to dense attention
    budget_mode: int = 0          # 0: window + fixed top-k, 1: entropy-derived budget,
                                  # 2: cumulative pooled mass
    budget_target: float = 0.0    # tau (mode 1: target retained fraction), theta (mode 2: mass)

    @property
    def N(self) -> int:
        return self.T * self.Hs * self.Ws

    @property
    def tile_grid(self) -> tuple[int, int, int]:
        e = TILE_EDGE
        return (-(-self.T // e), -(-self.Hs // e), -(-self.Ws // e))

    @property
    def NT(self) -> int:
        a, b, c = self.tile_grid
        return a * b * c

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the benchmark set, plus two small, genuinely sparse grids used by
# the parity tests (the 4x8x8 grid has only 4 tiles, so a radius-1 cube covers all of it).
WORKLOADS: dict[str, Workload] = {
    "tiny": Workload("tiny", B=1, H=2, d=64, T=4, Hs=8, Ws=8, seed=1000,
                     window_kind=0, radius=1, topk=1, dense_fraction=0.25),
    "wan13b": Workload("wan13b", B=1, H=12, d=128, T=21, Hs=30, Ws=52, seed=1001,
                       window_kind=1, radius=2, topk=8, dense_fraction=0.2),
    "wan5b": Workload("wan5b", B=1, H=24, d=128, T=31, Hs=22, Ws=40, seed=1002,
                      sink_frac=0.02, window_kind=0, radius=2, topk=8, dense_fraction=0.2),
    "wan14b": Workload("wan14b", B=1, H=40, d=128, T=21, Hs=45, Ws=80, seed=1003,
                       window_kind=0, radius=2, topk=16, dense_fraction=0.2),
    "hunyuan": Workload("hunyuan", B=1, H=24, d=128, T=33, Hs=45, Ws=80, seed=1004,
                        window_kind=1, radius=0, topk=0, dense_fraction=0.0,
                        budget_mode=1, budget_target=0.19),
    "tiny_s": Workload("tiny_s", B=1, H=2, d=64, T=8, Hs=16, Ws=16, seed=1000,
                       window_kind=0, radius=1, topk=1, dense_fraction=0.25),
    "tiny_ragged": Workload("tiny_ragged", B=1, H=2, d=64, T=6, Hs=10, Ws=9, seed=1000,
                            window_kind=0, radius=1, topk=1, dense_fraction=0.25),
}

WAN5B_RHO_SWEEP = (0.0, 0.1, 0.2, 0.4, 1.0)
HUNYUAN_TAU_SWEEP = (0.09, 0.14, 0.19)


def _features(T: int, Hs: int, Ws: int, phases: np.ndarray) -> np.ndarray:
    """[N, 19] float64 positional features in raster token order."""
    t = np.arange(T, dtype=np.float64) / T
    y = np.arange(Hs, dtype=np.float64) / Hs
    x = np.arange(Ws, dtype=np.float64) / Ws
    tt, yy, xx = np.meshgrid(t, y, x, indexing="ij")
    coords = [tt.reshape(-1), yy.reshape(-1), xx.reshape(-1)]
    cols = []
    for a in range(3):
        for fi, f in enumerate((1, 2, 3)):
            arg = 2.0 * math.pi * f * coords[a] + phases[a, fi]
            cols.append(np.sin(arg))
            cols.append(np.cos(arg))
    cols.append(np.ones_like(coords[0]))
    return np.stack(cols, axis=1)


def generate_qkv(w: Workload) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Q, K, V as CPU bfloat16 tensors of shape [B, N, H, d] (raster token order)."""
    rng = np.random.default_rng(w.seed)
    phases = rng.uniform(0.0, 2.0 * math.pi, size=(3, 3))
    feats = _features(w.T, w.Hs, w.Ws, phases).astype(np.float32)          # [N, 19]
    proj = [(rng.standard_normal((w.H, 19, w.d)) / math.sqrt(19.0)).astype(np.float32)
            for _ in range(3)]
    n_sink = int(math.floor(w.sink_frac * w.N + 0.5))
    out = []
    for p in proj:
        eps = rng.standard_normal((w.B, w.N, w.H, w.d), dtype=np.float32)
        base = (feats @ p.transpose(1, 0, 2).reshape(19, w.H * w.d)).reshape(w.N, w.H, w.d)
        x = eps
        x *= np.float32(w.noise_std)
        x += base[None]
        out.append(x)
    sinks = rng.choice(w.N, size=n_sink, replace=False) if n_sink > 0 else np.zeros(0, np.int64)
    tensors = []
    for x in out:
        if n_sink:
            x[:, sinks] *= np.float32(3.0)
        tensors.append(torch.from_numpy(x).to(torch.bfloat16))
    return tensors[0], tensors[1], tensors[2]


def generate_difficulty(w: Workload) -> torch.Tensor:
    """Per (batch item, query tile) difficulty in [0, 1), float32, shape [B, NQT]."""
    rng = np.random.default_rng(w.seed + 100)
    return torch.from_numpy(rng.random((w.B, w.NT)).astype(np.float32))


def sink_positions(w: Workload) -> np.ndarray:
    """The raster positions of the sink tokens drawn by generate_qkv (same stream)."""
    rng = np.random.default_rng(w.seed)
    rng.uniform(0.0, 2.0 * math.pi, size=(3, 3))
    for _ in range(3):
        rng.standard_normal((w.H, 19, w.d))
    for _ in range(3):
        rng.standard_normal((w.B, w.N, w.H, w.d), dtype=np.float32)
    n_sink = int(math.floor(w.sink_frac * w.N + 0.5))
    return rng.choice(w.N, size=n_sink, replace=False) if n_sink > 0 else np.zeros(0, np.int64)
