"""Stage 3 on the GPU against the oracle: per-dropped-block drift and the
drop-set drift J, with the GPU's own idx and lse.  Outputs start poisoned
(NaN), so an element the kernel skips cannot pass."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_global_mean_b200 import workloads
from tests.parity import assert_drift_close, np64, poison, sample_rows

pytestmark = pytest.mark.gpu


def _pipeline(ress, w, q, k, v, idx=None):
    n, h = q.shape[0], q.shape[1]
    nb = n // w.block
    if idx is None:
        idx = ress.ress_select_blocks(q, k, v if w.lam else None, w.budget, w.lam, w.block,
                                      idx=poison((h, nb, w.budget), torch.int32, q.device))
    budget = idx.shape[-1]
    out, lse = ress.ress_block_sparse_attn(q, k, v, idx, w.block,
                                           out=poison(q.shape, q.dtype, q.device),
                                           lse=poison((h, n), torch.float32, q.device))
    drift, jset = ress.ress_block_drift(
        q, k, v, idx, lse, w.block,
        drift=poison((h, nb, nb - budget), torch.float32, q.device),
        set_drift=poison((h, nb), torch.float32, q.device))
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


def test_64_heads_every_row(ress_gpu):
    H, nb, B, budget = 64, 6, 64, 2
    g = torch.Generator().manual_seed(64)
    q, k, v = (torch.randn(nb * B, H, 64, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    w = workloads.Workload("h64", 1, nb * B, nb * B, H, 64, "bf16", B, budget, 0.0, 0, "iid")
    idx, lse, drift, jset = _pipeline(ress_gpu, w, q, k, v)
    rows = [(h, i) for h in range(H) for i in range(nb)]
    _compare(q, k, v, idx, lse, drift, jset, B, rows)


@pytest.mark.parametrize("block", [64, 128])
def test_a_row_that_repeats_a_block_is_flagged(block, ress_gpu):
    """Drift rows must name distinct blocks: a repeat is flagged (detail 5)
    and every other row is still exact.  The planted row is made on the host
    and holds in-range indices only."""
    H, nb, budget = 1, 6, 3
    g = torch.Generator().manual_seed(block)
    q, k, v = (torch.randn(nb * block, H, 64, generator=g).to(torch.bfloat16).cuda()
               for _ in range(3))
    idx_np = np.tile(np.array([0, 2, 4], dtype=np.int32), (H, nb, 1))
    idx_np[0, 3] = [1, 1, 5]
    idx = torch.from_numpy(idx_np).cuda()
    out, lse = ress_gpu.ress_block_sparse_attn(q, k, v, idx, block)
    assert ress_gpu.ress_check_device_errors()[0] == 0          # attention accepts repeats
    drift = poison((H, nb, nb - budget), torch.float32)
    jset = poison((H, nb), torch.float32)
    ress_gpu.ress_block_drift(q, k, v, idx, lse, block, drift=drift, set_drift=jset)
    status, detail = ress_gpu.ress_check_device_errors()
    assert status == ress_gpu.RESS_ERR_BAD_INDEX and detail == 5
    rows = [(0, i) for i in range(nb) if i != 3]
    _compare(q, k, v, idx, lse, drift, jset, block, rows)
