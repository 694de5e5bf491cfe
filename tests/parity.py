"""Comparison helpers shared by the GPU parity tests (CUDA path vs the oracle).

Tolerances:
* mask: every (head, query block) row equals the oracle's kept set, except
  that a differing block is excused when its oracle score lies within 1e-4 of
  the oracle's budget-th score (the ranked quantity: the pooled logit when
  lambda == 0, which orders a row exactly as the probability does, and
  p + lambda * c otherwise);
* attention output (bf16 inputs) against the float64 oracle run with the GPU's
  own idx: max-abs-error <= 2e-2 and mean-abs-error <= 2e-3;
* lse: relative error <= 1e-3;
* drift and set drift: |gpu - ref| <= 2e-2 * ref + 1e-4 * max(ref) (the pages
  fix no tolerance for drift; this one follows from bf16 operands with fp32
  accumulation).
"""

from __future__ import annotations

import numpy as np
import torch

MASK_MARGIN = 1e-4
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
LSE_REL = 1e-3
DRIFT_REL = 2e-2
DRIFT_ABS_FRAC = 1e-4


def poison(shape, dtype, device="cuda") -> torch.Tensor:
    """An output buffer pre-filled with values no kernel writes (NaN for
    floating point, -1 for integers), so an element the kernel skips cannot
    pass by holding a plausible earlier result."""
    if dtype.is_floating_point:
        return torch.full(shape, float("nan"), dtype=dtype, device=device)
    return torch.full(shape, -1, dtype=dtype, device=device)


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def sample_rows(heads: int, nb: int, count: int = 64, seed: int = 1234):
    """Seeded (h, i) sample plus the first and last query block of every head."""
    rng = np.random.default_rng(seed)
    rows = {(h, 0) for h in range(heads)} | {(h, nb - 1) for h in range(heads)}
    while len(rows) < 2 * heads + count and len(rows) < heads * nb:
        rows.add((int(rng.integers(heads)), int(rng.integers(nb))))
    return sorted(rows)


def mask_mismatch(idx_gpu: np.ndarray, idx_ref: np.ndarray, ranked: np.ndarray, budget: int):
    """Returns (rows that differ, rows not excused by the margin rule)."""
    h_count, nb, _ = idx_ref.shape
    differ, bad = 0, []
    for h in range(h_count):
        for i in range(nb):
            a = set(idx_gpu[h, i].tolist())
            b = set(idx_ref[h, i].tolist())
            if a == b:
                continue
            differ += 1
            row = ranked[h, i]
            kth = np.sort(row)[::-1][budget - 1]
            for j in a ^ b:
                if not (0 <= j < nb) or abs(row[j] - kth) > MASK_MARGIN:
                    bad.append((h, i, j))
                    break
    return differ, bad


def assert_mask_parity(idx_gpu, idx_ref, ranked, budget, max_excused_frac=0.05):
    g = idx_gpu if isinstance(idx_gpu, np.ndarray) else idx_gpu.cpu().numpy()
    assert g.shape == idx_ref.shape
    # ascending, in range, distinct
    assert np.all(np.diff(g, axis=-1) > 0), "rows must be strictly ascending"
    differ, bad = mask_mismatch(g, idx_ref, ranked, budget)
    assert not bad, f"{len(bad)} rows differ beyond the 1e-4 margin, e.g. {bad[:5]}"
    assert differ <= max_excused_frac * g.shape[0] * g.shape[1], f"{differ} excused rows"
    return differ


def assert_attn_close(out_gpu: np.ndarray, out_ref: np.ndarray, lse_gpu=None, lse_ref=None):
    err = np.abs(out_gpu - out_ref)
    assert np.isfinite(out_gpu).all()
    assert err.max() <= ATTN_MAX_ABS, f"max abs err {err.max():.3e}"
    assert err.mean() <= ATTN_MEAN_ABS, f"mean abs err {err.mean():.3e}"
    if lse_gpu is not None:
        rel = np.abs(lse_gpu - lse_ref) / np.maximum(np.abs(lse_ref), 1e-6)
        assert rel.max() <= LSE_REL, f"lse rel err {rel.max():.3e}"
    return float(err.max()), float(err.mean())


def assert_drift_close(gpu: np.ndarray, ref: np.ndarray):
    assert gpu.shape == ref.shape
    if ref.size == 0:
        return 0.0
    assert np.isfinite(gpu).all()
    scale = float(np.max(np.abs(ref)))
    err = np.abs(gpu - ref)
    bound = DRIFT_REL * np.abs(ref) + DRIFT_ABS_FRAC * scale
    worst = float(np.max(err / np.maximum(bound, 1e-30)))
    assert np.all(err <= bound), f"drift error exceeds bound by {worst:.2f}x"
    return worst
