"""Stage 3 on the GPU against the oracle: per-dropped-block drift and the
drop-set drift J, with the GPU's own idx and lse."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_global_mean_b200 import workloads
from tests.parity import assert_drift_close, np64, sample_rows

pytestmark = pytest.mark.gpu


def _pipeline(ress, w, q, k, v, idx=None):
    if idx is None:
        idx = ress.ress_select_blocks(q, k, v if w.lam else None, w.budget, w.lam, w.block)
    out, lse = ress.ress_block_sparse_attn(q, k, v, idx, w.block)
    drift, jset = ress.ress_block_drift(q, k, v, idx, lse, w.block)
    status, detail = ress.ress_check_device_errors()
    assert status == 0, (status, detail)
    return idx, lse, drift, jset


def _compare(q, k, v, idx, lse, drift, jset, block, rows):
    ref_d, ref_j = oracle.block_drift(np64(q), np64(k), np64(v), idx.cpu().numpy(), np64(lse),
                                      block, rows=rows)
    hs = np.array([r[0] for r in rows])
    is_ = np.array([r[1] for r in rows])
    assert_drift_close(np64(drift)[hs, is_], ref_d[hs, is_])
    assert_drift_close(np64(jset)[hs, is_], ref_j[hs, is_])


@pytest.mark.parametrize("name", ["tiny", "vggt8"])
def test_every_row_block64(name, ress_gpu, wcache):
    w = workloads.WORKLOADS[name]
    q, k, v = wcache.get(w)
    idx, lse, drift, jset = _pipeline(ress_gpu, w, q, k, v)
    rows = [(h, i) for h in range(w.heads) for i in range(w.n_blocks)]
    _compare(q, k, v, idx, lse, drift, jset, w.block, rows)


def test_every_row_block128_eight_views(ress_gpu, wcache):
    w = workloads.scaled(workloads.WORKLOADS["views200"], 8)
    q, k, v = wcache.get(w)
    idx, lse, drift, jset = _pipeline(ress_gpu, w, q, k, v)
    rows = [(h, i) for h in range(w.heads) for i in range(w.n_blocks)]
    _compare(q, k, v, idx, lse, drift, jset, w.block, rows)


def test_sampled_rows_views200(ress_gpu, wcache):
    w = workloads.WORKLOADS["views200"]
    q, k, v = wcache.get(w)
    idx, lse, drift, jset = _pipeline(ress_gpu, w, q, k, v)
    rows = sample_rows(w.heads, w.n_blocks, count=8)[:24]
    _compare(q, k, v, idx, lse, drift, jset, w.block, rows)


@pytest.mark.parametrize("block,nb,budget", [(64, 7, 2), (64, 9, 9), (128, 5, 1), (128, 6, 6)])
def test_odd_sizes_and_empty_drop_sets(block, nb, budget, ress_gpu):
    H = 2
    g = torch.Generator().manual_seed(nb + 10 * budget)
    q, k, v = (torch.randn(nb * block, H, 64, generator=g).to(torch.bfloat16).cuda()
               for _ in range(3))
    rng = np.random.default_rng(budget)
    idx_np = np.stack([np.stack([np.sort(rng.choice(nb, budget, replace=False))
                                 for _ in range(nb)]) for _ in range(H)]).astype(np.int32)
    w = workloads.Workload("odd", 1, nb * block, nb * block, H, 64, "bf16", block, budget, 0.0, 0,
                           "iid")
    idx = torch.from_numpy(idx_np).cuda()
    _, lse, drift, jset = _pipeline(ress_gpu, w, q, k, v, idx)
    assert drift.shape == (H, nb, nb - budget)
    if budget == nb:
        assert torch.all(jset == 0)
    rows = [(h, i) for h in range(H) for i in range(nb)]
    _compare(q, k, v, idx, lse, drift, jset, block, rows)
