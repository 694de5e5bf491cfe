"""Seeded synthetic multi-view token workloads.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no pooling, scoring, selection or attention).  Both the
CUDA path and the CPU oracle are fed from it.

The workloads stand in for the VGGT global-attention inputs that the ReSS and
VASC pages measure on (ScanNet++, NeuralRGB-D and DTU at up to 100 views,
ReSS Table 1 and Table S7; VASC section 5.2).  Those datasets and the trained
VGGT weights are not available, so the token statistics are synthetic:

* a VGGT view holds 1,374 tokens (1 camera + 4 register + 37x37 patch tokens)
  and is zero-padded to 1,408 tokens, a multiple of both block sizes;
* every (tensor in {Q, K, V}, view, head) draws a cluster mean mu ~ N(0, I_64)
  and each real token is mu + 0.5 * N(0, I_64) (noise standard deviation 0.5);
* padding tokens are exact zero vectors in Q, K and V;
* optional per-head cluster scales a_h ~ U[0.5, 2] (shared by Q, K and V);
* optional outlier tokens: a seeded 5 % of the real token positions (the same
  positions for Q, K, V and every head) have their whole vector multiplied by 4.

Tensors are token-major ``[N, H, d]`` (one token row is H*d contiguous values).
Values are drawn in fp32 and rounded to bf16 (round to nearest even) for the
bf16 workloads; the tiny workload stays fp32 with iid N(0, 1) entries.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch

TOKENS_PER_VIEW_REAL = 1374     # 1 camera + 4 register + 37 * 37 patches
TOKENS_PER_VIEW_PADDED = 1408   # 22 blocks of 64, 11 blocks of 128


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, selection knobs and the generator recipe."""

    name: str
    views: int
    tokens_per_view: int          # padded tokens per view
    real_tokens_per_view: int     # tokens that carry data; the rest are zero
    heads: int
    head_dim: int
    dtype: str                    # "bf16" or "f32"
    block: int                    # B: tokens per query block and per key block
    budget: int                   # k: kept key blocks per query block
    lam: float                    # weight of the value-contrast term
    seed: int
    generator: str                # "iid" or "cluster"
    head_scale: bool = False      # per-head cluster scales a_h ~ U[0.5, 2]
    outlier_frac: float = 0.0     # fraction of real token positions scaled
    outlier_scale: float = 1.0
    drift: bool = False           # the drift stage is part of this workload

    @property
    def n_tokens(self) -> int:
        return self.views * self.tokens_per_view

    @property
    def n_blocks(self) -> int:
        return self.n_tokens // self.block

    @property
    def sparsity(self) -> float:
        """Measured sparsity of any exact-budget mask: 1 - k / nb."""
        return 1.0 - self.budget / self.n_blocks

    def effective_flops(self) -> float:
        """4 * N * kept_keys * d * H: the kept-key attention work (QK^T and PV)."""
        return 4.0 * self.n_tokens * (self.budget * self.block) * self.head_dim * self.heads

    def dense_flops(self) -> float:
        return 4.0 * self.n_tokens * self.n_tokens * self.head_dim * self.heads

    def drift_flops(self) -> float:
        """4 * N * (nb - k) * B * d * H: the work over every dropped key block."""
        return 4.0 * self.n_tokens * ((self.n_blocks - self.budget) * self.block) * self.head_dim * self.heads


WORKLOADS = {
    # 2 views x 256 tokens, H=2, fp32 iid N(0,1), 8 key blocks, keep 4.
    "tiny": Workload("tiny", views=2, tokens_per_view=256, real_tokens_per_view=256, heads=2,
                     head_dim=64, dtype="f32", block=64, budget=4, lam=0.0, seed=0,
                     generator="iid"),
    # 8 VGGT views, 50 % of 176 key blocks kept.
    "vggt8": Workload("vggt8", views=8, tokens_per_view=TOKENS_PER_VIEW_PADDED,
                      real_tokens_per_view=TOKENS_PER_VIEW_REAL, heads=16, head_dim=64,
                      dtype="bf16", block=64, budget=88, lam=0.0, seed=1, generator="cluster"),
    # 32 views, 75 % sparsity (176 of 704 kept), value contrast weight 0.5.
    "views32": Workload("views32", views=32, tokens_per_view=TOKENS_PER_VIEW_PADDED,
                        real_tokens_per_view=TOKENS_PER_VIEW_REAL, heads=16, head_dim=64,
                        dtype="bf16", block=64, budget=176, lam=0.5, seed=2,
                        generator="cluster", head_scale=True),
    # 100 views, 90 % sparsity (220 of 2,200 kept), 5 % outliers with 4x norm.
    "views100": Workload("views100", views=100, tokens_per_view=TOKENS_PER_VIEW_PADDED,
                         real_tokens_per_view=TOKENS_PER_VIEW_REAL, heads=16, head_dim=64,
                         dtype="bf16", block=64, budget=220, lam=0.0, seed=3,
                         generator="cluster", outlier_frac=0.05, outlier_scale=4.0),
    # 200 views, block 128, 95 % sparsity (110 of 2,200 kept), drift stage on.
    "views200": Workload("views200", views=200, tokens_per_view=TOKENS_PER_VIEW_PADDED,
                         real_tokens_per_view=TOKENS_PER_VIEW_REAL, heads=16, head_dim=64,
                         dtype="bf16", block=128, budget=110, lam=0.0, seed=4,
                         generator="cluster", drift=True),
}


def scaled(w: Workload, views: int, budget: Optional[int] = None, name: Optional[str] = None,
           seed: Optional[int] = None) -> Workload:
    """The same recipe with fewer views (for quick cases that still span many tiles)."""
    nb = views * w.tokens_per_view // w.block
    if budget is None:
        budget = max(1, round(w.budget * nb / w.n_blocks))
    return dataclasses.replace(w, name=name or f"{w.name}@{views}v", views=views,
                               budget=budget, seed=w.seed if seed is None else seed)


def generate(w: Workload, device: str = "cpu", seed: Optional[int] = None):
    """Return (q, k, v) as ``[N, H, d]`` tensors of the workload's dtype.

    Random numbers come from one ``torch.Generator`` on the CPU seeded with
    ``seed`` (default: the workload's seed), drawn in a fixed order, so the
    result depends only on the recipe and the seed.
    """
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    N, H, d = w.n_tokens, w.heads, w.head_dim
    if w.generator == "iid":
        out = [torch.randn(N, H, d, generator=g, dtype=torch.float32) for _ in range(3)]
        if w.dtype == "bf16":
            out = [t.to(torch.bfloat16) for t in out]
        return tuple(t.to(device) for t in out)

    assert w.generator == "cluster"
    V, T, R = w.views, w.tokens_per_view, w.real_tokens_per_view
    mu = torch.randn(3, V, H, d, generator=g, dtype=torch.float32)
    if w.head_scale:
        a = 0.5 + 1.5 * torch.rand(H, generator=g, dtype=torch.float32)
        mu = mu * a.view(1, 1, H, 1)
    scale = None
    if w.outlier_frac > 0.0:
        n_pos = V * R
        n_out = int(round(w.outlier_frac * n_pos))
        pos = torch.randperm(n_pos, generator=g)[:n_out]
        scale = torch.ones(n_pos, dtype=torch.float32)
        scale[pos] = w.outlier_scale
        scale = scale.view(V, R, 1, 1)
    out_dtype = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    tensors = []
    for t in range(3):
        x = torch.randn(V, R, H, d, generator=g, dtype=torch.float32)
        x.mul_(0.5).add_(mu[t].view(V, 1, H, d))
        if scale is not None:
            x.mul_(scale)
        full = torch.zeros(V, T, H, d, dtype=out_dtype)
        full[:, :R] = x.to(out_dtype)
        del x
        tensors.append(full.view(V * T, H, d).to(device))
    return tuple(tensors)
