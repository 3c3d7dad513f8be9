"""Seeded synthetic Q/K/V for video-DiT-shaped self-attention.

This module is the one piece shared by the CUDA path's tests/bench and the
CPU oracle's tests.  It holds none of the attention method's arithmetic: it
only draws inputs.  The pages measure on Wan2.1 and HunyuanVideo activations
(AB-Attention page, section "Performans Sonuçları ve Pratik Çıkarımlar"); no
model weights are available, so these inputs stand in for them at the same
shapes.

Recipe (per batch element b and head h, tokens on a T x Y x X grid in raster
order l = (t*Y + y)*X + x, normalised position p = (t/T, y/Y, x/X)):

* a shared projection W in R^{F x d}, entries N(0, alpha^2) with
  alpha^2 = s_peak / (sqrt(d) * F), s_peak = 8 (so q.k/sqrt(d) of two
  tokens at the same position is about s_peak);
* a per-head length scale ell_h = 2^(1 + 3U) tokens, U ~ U[0,1);
* per-head frequencies omega_f in R^3 with omega_{f,a} ~ N(0, (N_a/ell_h)^2),
  N = (T, Y, X), and phases phi_f ~ U[0, 2 pi), f = 1..F;
* features Phi_f(p) = sqrt(2) cos(omega_f . p + phi_f);
* Q = Phi W + 0.5 N(0,1), K = Phi W + 0.5 N(0,1) (independent noise);
* V ~ N(0,1), and each token's V row is scaled by 10 with probability 0.01;
* every tensor is rounded to bfloat16 (round-to-nearest-even).

All draws come from one ``torch.Generator`` seeded with ``seed``, in a fixed
order: W, then for each (b, h): U, omega, phi, Q noise, K noise, V, outlier
mask.  The same seed gives the same tensors on any machine with this torch.

Cross-attention (queries from one sequence, keys and values from another:
Cross-Attention glossary page, "Cross-Attention Nasıl Çalışır?"): the queries
live on a grid (T, Y, X) and the keys and values on a second grid
(T', Y', X') covering the same normalised space, e.g. a clip attending to a
shorter or longer reference clip.  Both sides use the same per-head features
Phi (same omega, phi), each at its own positions; the draw order is the
same, with the K noise, V and outlier mask drawn for the L' key tokens.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

DATA_SEED = 1234
SAMPLER_SEED = 42


@dataclass(frozen=True)
class Workload:
    """A named attention workload: shapes and method parameters."""

    name: str
    B: int
    H: int
    grid: tuple  # (T, Y, X)
    d: int
    F: int
    q_block: int
    kv_block: int
    C: int
    keep_ratio: float
    kmeans_iters: int = 3
    extra: dict = field(default_factory=dict)
    grid_kv: tuple | None = None  # key/value grid under cross-attention (None: self-attention)

    @property
    def L(self) -> int:
        T, Y, X = self.grid
        return T * Y * X

    @property
    def Lk(self) -> int:
        if self.grid_kv is None:
            return self.L
        T, Y, X = self.grid_kv
        return T * Y * X

    @property
    def Nq(self) -> int:
        return -(-self.L // self.q_block)

    @property
    def Nkv(self) -> int:
        return -(-self.Lk // self.kv_block)

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


# Workloads: the tiny case the oracle runs in full, a small video, the
# Wan2.1-480p / HunyuanVideo-720p / Wan-720p self-attention shapes, and
# cross-attention cases (a clip attending to a shorter / a longer clip, ragged
# key counts: 3330 keys is not a multiple of 8; the Wan2.1-480p clip attending
# to a 9-frame reference clip).
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, (4, 16, 16), 64, 8, 64, 16, 4, 0.10),
    "small": Workload("small", 1, 4, (8, 32, 32), 128, 16, 128, 16, 8, 0.10),
    "wan480": Workload("wan480", 1, 40, (21, 30, 52), 128, 16, 128, 16, 8, 0.11),
    "hunyuan720": Workload("hunyuan720", 1, 24, (33, 45, 80), 128, 16, 128, 16, 8, 0.08),
    "wan720": Workload("wan720", 1, 40, (21, 45, 80), 128, 16, 128, 16, 8, 0.10),
    "cross_short": Workload("cross_short", 1, 3, (8, 32, 32), 128, 16, 128, 16, 8, 0.10,
                            grid_kv=(3, 30, 37)),
    "cross_long": Workload("cross_long", 2, 2, (3, 20, 30), 64, 8, 64, 32, 4, 0.15,
                           grid_kv=(9, 24, 40)),
    # the Wan2.1-480p clip attending to a 9-frame reference clip of the same frame size
    "cross_wan480": Workload("cross_wan480", 1, 40, (21, 30, 52), 128, 16, 128, 16, 8, 0.11,
                             grid_kv=(9, 30, 52)),
}


def positions(grid) -> torch.Tensor:
    """Normalised (t/T, y/Y, x/X) for every token in raster order, [L, 3] fp64."""
    T, Y, X = grid
    t = torch.arange(T, dtype=torch.float64) / T
    y = torch.arange(Y, dtype=torch.float64) / Y
    x = torch.arange(X, dtype=torch.float64) / X
    tt, yy, xx = torch.meshgrid(t, y, x, indexing="ij")
    return torch.stack([tt.reshape(-1), yy.reshape(-1), xx.reshape(-1)], dim=1)


def make_qkv(B: int, H: int, grid, d: int, F: int, seed: int = DATA_SEED,
             s_peak: float = 8.0, noise: float = 0.5, outlier_p: float = 0.01,
             outlier_scale: float = 10.0):
    """Q, K, V as contiguous bfloat16 CPU tensors of shape [B, H, L, d]."""
    g = torch.Generator().manual_seed(int(seed))
    T, Y, X = grid
    L = T * Y * X
    pos = positions(grid)                                   # [L, 3]
    alpha = math.sqrt(s_peak / (math.sqrt(d) * F))
    W = torch.randn(F, d, generator=g, dtype=torch.float64) * alpha
    N = torch.tensor([T, Y, X], dtype=torch.float64)
    Q = torch.empty(B, H, L, d, dtype=torch.bfloat16)
    K = torch.empty(B, H, L, d, dtype=torch.bfloat16)
    V = torch.empty(B, H, L, d, dtype=torch.bfloat16)
    for b in range(B):
        for h in range(H):
            u = torch.rand(1, generator=g, dtype=torch.float64).item()
            ell = 2.0 ** (1.0 + 3.0 * u)
            omega = torch.randn(F, 3, generator=g, dtype=torch.float64) * (N / ell)
            phi = torch.rand(F, generator=g, dtype=torch.float64) * (2.0 * math.pi)
            feats = math.sqrt(2.0) * torch.cos(pos @ omega.T + phi)   # [L, F]
            base = (feats @ W).to(torch.float32)                   # [L, d]
            qn = torch.randn(L, d, generator=g)
            kn = torch.randn(L, d, generator=g)
            v = torch.randn(L, d, generator=g)
            out = torch.rand(L, generator=g) < outlier_p
            Q[b, h] = (base + noise * qn).to(torch.bfloat16)
            K[b, h] = (base + noise * kn).to(torch.bfloat16)
            v[out] *= outlier_scale
            V[b, h] = v.to(torch.bfloat16)
    return Q, K, V


def make_cross_qkv(B: int, H: int, grid, grid_kv, d: int, F: int, seed: int = DATA_SEED,
                   s_peak: float = 8.0, noise: float = 0.5, outlier_p: float = 0.01,
                   outlier_scale: float = 10.0):
    """Cross-attention inputs: Q [B, H, L, d] on ``grid``, K and V
    [B, H, Lk, d] on ``grid_kv`` (contiguous bfloat16 CPU tensors)."""
    g = torch.Generator().manual_seed(int(seed))
    T, Y, X = grid
    L = T * Y * X
    Lk = grid_kv[0] * grid_kv[1] * grid_kv[2]
    pos_q, pos_k = positions(grid), positions(grid_kv)
    alpha = math.sqrt(s_peak / (math.sqrt(d) * F))
    W = torch.randn(F, d, generator=g, dtype=torch.float64) * alpha
    N = torch.tensor([T, Y, X], dtype=torch.float64)
    Q = torch.empty(B, H, L, d, dtype=torch.bfloat16)
    K = torch.empty(B, H, Lk, d, dtype=torch.bfloat16)
    V = torch.empty(B, H, Lk, d, dtype=torch.bfloat16)
    for b in range(B):
        for h in range(H):
            u = torch.rand(1, generator=g, dtype=torch.float64).item()
            ell = 2.0 ** (1.0 + 3.0 * u)
            omega = torch.randn(F, 3, generator=g, dtype=torch.float64) * (N / ell)
            phi = torch.rand(F, generator=g, dtype=torch.float64) * (2.0 * math.pi)
            base_q = (math.sqrt(2.0) * torch.cos(pos_q @ omega.T + phi) @ W).to(torch.float32)
            base_k = (math.sqrt(2.0) * torch.cos(pos_k @ omega.T + phi) @ W).to(torch.float32)
            qn = torch.randn(L, d, generator=g)
            kn = torch.randn(Lk, d, generator=g)
            v = torch.randn(Lk, d, generator=g)
            out = torch.rand(Lk, generator=g) < outlier_p
            Q[b, h] = (base_q + noise * qn).to(torch.bfloat16)
            K[b, h] = (base_k + noise * kn).to(torch.bfloat16)
            v[out] *= outlier_scale
            V[b, h] = v.to(torch.bfloat16)
    return Q, K, V


def make_workload_qkv(w: Workload, seed: int = DATA_SEED):
    if w.grid_kv is not None:
        return make_cross_qkv(w.B, w.H, w.grid, w.grid_kv, w.d, w.F, seed=seed)
    return make_qkv(w.B, w.H, w.grid, w.d, w.F, seed=seed)
