"""The seeded synthetic inputs follow their stated recipe: shapes and dtypes,
exact-zero padding, per-view clusters with noise of standard deviation 0.5,
outlier positions shared by Q, K, V and every head, per-head cluster scales
in [0.5, 2], and determinism in the seed."""

import numpy as np
import torch

from block_sparse_global_mean_b200 import workloads

W = workloads.WORKLOADS


def test_shapes_dtypes_and_budgets_of_every_workload():
    expect = {"tiny": (512, 2, torch.float32, 64, 4), "vggt8": (11264, 16, torch.bfloat16, 64, 88),
              "views32": (45056, 16, torch.bfloat16, 64, 176),
              "views100": (140800, 16, torch.bfloat16, 64, 220),
              "views200": (281600, 16, torch.bfloat16, 128, 110)}
    for name, (n, h, dtype, block, budget) in expect.items():
        w = W[name]
        assert (w.n_tokens, w.heads, w.block, w.budget) == (n, h, block, budget)
        assert w.n_tokens % w.block == 0
        small = workloads.scaled(w, 1) if w.generator == "cluster" else w
        q, k, v = workloads.generate(small)
        assert q.shape == (small.n_tokens, h, 64) and q.dtype == dtype
        assert k.shape == q.shape and v.shape == q.shape
    assert W["views100"].sparsity == 0.9 and W["views200"].sparsity == 0.95


def test_padding_is_exactly_zero_and_real_tokens_are_not():
    w = workloads.scaled(W["vggt8"], 3)
    for x in workloads.generate(w):
        x = x.view(w.views, w.tokens_per_view, w.heads, 64)
        assert (x[:, w.real_tokens_per_view:] == 0).all()
        assert (x[:, :w.real_tokens_per_view].float().abs().sum(-1) > 0).all()


def test_clusters_have_noise_std_half_around_a_unit_normal_mean():
    w = workloads.scaled(W["vggt8"], 4)
    q, _, _ = workloads.generate(w)
    x = q.float().view(w.views, w.tokens_per_view, w.heads, 64)[:, :w.real_tokens_per_view]
    mean = x.mean(dim=1, keepdim=True)                   # ~ mu (per view, head)
    resid = (x - mean).std().item()
    assert abs(resid - 0.5) < 0.01
    assert abs(mean.std().item() - 1.0) < 0.1


def test_outliers_are_five_percent_shared_by_q_k_v_and_heads():
    w = workloads.scaled(W["views100"], 3)
    q, k, v = (t.float().view(w.views, w.tokens_per_view, w.heads, 64)[:, :w.real_tokens_per_view]
               for t in workloads.generate(w))
    flags = []
    for x in (q, k, v):
        mean = x.mean(dim=1, keepdim=True)
        dev = (x - mean).norm(dim=-1)                    # [V, R, H]
        flags.append(dev > 2.5 * dev.median())           # outliers deviate by ~4x
    for f in flags[1:]:
        assert torch.equal(f, flags[0])                  # same positions in Q, K, V
    f = flags[0]
    assert (f == f[:, :, :1]).all()                      # same positions in every head
    frac = f[:, :, 0].float().mean().item()
    assert abs(frac - 0.05) < 0.005


def test_head_scales_lie_in_half_to_two():
    w = workloads.scaled(W["views32"], 6)
    q, _, _ = workloads.generate(w)
    x = q.float().view(w.views, w.tokens_per_view, w.heads, 64)[:, :w.real_tokens_per_view]
    mu = x.mean(dim=1)                                   # [V, H, d]
    rms = mu.pow(2).mean(dim=(0, 2)).sqrt()              # ~ a_h per head
    assert (rms > 0.4).all() and (rms < 2.2).all()
    assert rms.max() / rms.min() > 1.3                   # the scales differ across heads


def test_generation_is_deterministic_in_the_seed():
    w = workloads.scaled(W["vggt8"], 1)
    a = workloads.generate(w)
    b = workloads.generate(w)
    c = workloads.generate(w, seed=w.seed + 1000)
    for x, y, z in zip(a, b, c):
        assert torch.equal(x, y)
        assert not torch.equal(x, z)
    t1 = workloads.generate(W["tiny"])[0]
    assert abs(t1.mean().item()) < 0.02 and abs(t1.std().item() - 1.0) < 0.02
