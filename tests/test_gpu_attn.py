"""Stage 2 on the GPU against the oracle (run with the GPU's own idx): every
row at the small sizes, sampled rows at the full sizes, and the edge cases
(full budget = dense attention, budget 1, an odd number of query blocks,
unsorted and duplicated indices, out-of-range indices, one head and the
64-head maximum, a grid near the 10,000-block limit).  Outputs start
poisoned (NaN), so an element the kernel skips cannot pass."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_global_mean_b200 import workloads
from tests.parity import assert_attn_close, np64, poison, sample_rows

pytestmark = pytest.mark.gpu


def _run(ress, w, q, k, v, idx, out_dtype=None):
    n, h = q.shape[0], q.shape[1]
    out = poison(q.shape, out_dtype or q.dtype, q.device)
    lse = poison((h, n), torch.float32, q.device)
    out, lse = ress.ress_block_sparse_attn(q, k, v, idx, w.block, out=out, lse=lse)
    status, detail = ress.ress_check_device_errors()
    assert status == 0, (status, detail)
    return out, lse


def _compare_rows(q, k, v, idx_np, out, lse, block, rows):
    qn, kn, vn = np64(q), np64(k), np64(v)
    ref_o, ref_l = oracle.sparse_attention(qn, kn, vn, idx_np, block, rows=rows)
    sel = np.zeros(ref_o.shape[:2], dtype=bool)
    for h, i in rows:
        sel[i * block:(i + 1) * block, h] = True
    got_o = np64(out)
    got_l = np64(lse)
    return assert_attn_close(got_o[sel], ref_o[sel], got_l.T[sel], ref_l.T[sel])


@pytest.mark.parametrize("name", ["tiny", "vggt8"])
def test_every_row_matches_oracle(name, ress_gpu, wcache):
    w = workloads.WORKLOADS[name]
    q, k, v = wcache.get(w)
    idx = ress_gpu.ress_select_blocks(q, k, v if w.lam else None, w.budget, w.lam, w.block)
    out, lse = _run(ress_gpu, w, q, k, v, idx)
    assert out.dtype == q.dtype
    rows = [(h, i) for h in range(w.heads) for i in range(w.n_blocks)]
    _compare_rows(q, k, v, idx.cpu().numpy(), out, lse, w.block, rows)


@pytest.mark.parametrize("name", ["views32", "views100", "views200"])
def test_sampled_rows_at_full_size(name, ress_gpu, wcache):
    """The kernel and launch configuration the benchmark times, with a float32
    output so that the comparison measures the kernel's arithmetic (a bf16
    output cannot hold |O| >= 8 within 2e-2: half an ulp there is >= 1/32)."""
    w = workloads.WORKLOADS[name]
    q, k, v = wcache.get(w)
    idx = ress_gpu.ress_select_blocks(q, k, v if w.lam else None, w.budget, w.lam, w.block)
    out, lse = _run(ress_gpu, w, q, k, v, idx, out_dtype=torch.float32)
    rows = sample_rows(w.heads, w.n_blocks)
    _compare_rows(q, k, v, idx.cpu().numpy(), out, lse, w.block, rows)
    assert torch.isfinite(out).all()
    # The bf16 output is the float32 result rounded to nearest.
    out16, _ = _run(ress_gpu, w, q, k, v, idx)
    assert torch.equal(out16, out.to(torch.bfloat16))


def _random_idx(H, nb, budget, seed, dup=False, shuffle=False):
    rng = np.random.default_rng(seed)
    idx = np.stack([np.stack([np.sort(rng.choice(nb, budget, replace=False)) for _ in range(nb)])
                    for _ in range(H)]).astype(np.int32)
    if dup:
        idx[..., -1] = idx[..., 0]
    if shuffle:
        for h in range(H):
            for i in range(nb):
                rng.shuffle(idx[h, i])
    return idx


@pytest.mark.parametrize("block,nb,budget", [(64, 7, 7), (64, 7, 1), (64, 9, 3), (128, 6, 2),
                                             (128, 5, 5), (64, 40, 13)])
def test_random_masks_odd_sizes(block, nb, budget, ress_gpu):
    H = 3
    g = torch.Generator().manual_seed(nb * 100 + budget)
    q, k, v = (torch.randn(nb * block, H, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    idx = _random_idx(H, nb, budget, seed=budget)
    w = workloads.Workload("rand", 1, nb * block, nb * block, H, 64, "bf16", block, budget, 0.0, 0,
                           "iid")
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out, lse = _run(ress_gpu, w, qd, kd, vd, torch.from_numpy(idx).cuda())
    rows = [(h, i) for h in range(H) for i in range(nb)]
    _compare_rows(q, k, v, idx, out.cpu(), lse.cpu(), block, rows)


def test_full_budget_equals_dense_attention(ress_gpu):
    H, nb, B = 2, 16, 64
    g = torch.Generator().manual_seed(3)
    q, k, v = (torch.randn(nb * B, H, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    idx = np.tile(np.arange(nb, dtype=np.int32), (H, nb, 1))
    w = workloads.Workload("dense", 1, nb * B, nb * B, H, 64, "bf16", B, nb, 0.0, 0, "iid")
    out, lse = _run(ress_gpu, w, q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(idx).cuda())
    qn, kn, vn = np64(q), np64(k), np64(v)
    for h in range(H):
        s = qn[:, h] @ kn[:, h].T / 8.0
        p = np.exp(s - s.max(1, keepdims=True))
        ref = (p / p.sum(1, keepdims=True)) @ vn[:, h]
        assert_attn_close(np64(out)[:, h], ref)


def test_unsorted_and_duplicated_indices_count_once(ress_gpu):
    H, nb, B, budget = 2, 10, 64, 5
    g = torch.Generator().manual_seed(4)
    q, k, v = (torch.randn(nb * B, H, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    idx = _random_idx(H, nb, budget, seed=9, dup=True, shuffle=True)
    w = workloads.Workload("dup", 1, nb * B, nb * B, H, 64, "bf16", B, budget, 0.0, 0, "iid")
    out, lse = _run(ress_gpu, w, q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(idx).cuda())
    qn, kn, vn = np64(q), np64(k), np64(v)
    for h in range(H):
        for i in range(nb):
            kept = sorted(set(idx[h, i].tolist()))
            ref_o, ref_l = oracle.sparse_attention_block(qn, kn, vn, kept, h, i, B)
            assert_attn_close(np64(out)[i * B:(i + 1) * B, h], ref_o,
                              np64(lse)[h, i * B:(i + 1) * B], ref_l)


def test_out_of_range_indices_are_skipped_and_flagged(ress_gpu):
    H, nb, B, budget = 1, 6, 64, 3
    g = torch.Generator().manual_seed(6)
    q, k, v = (torch.randn(nb * B, H, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    idx = np.tile(np.array([0, 2, 4], dtype=np.int32), (H, nb, 1))
    idx[0, 1, 2] = 77          # out of range
    idx[0, 3, 0] = -5          # out of range
    out, lse = ress_gpu.ress_block_sparse_attn(q.cuda(), k.cuda(), v.cuda(),
                                               torch.from_numpy(idx).cuda(), B,
                                               out=poison((nb * B, H, 64), torch.bfloat16),
                                               lse=poison((H, nb * B), torch.float32))
    status, detail = ress_gpu.ress_check_device_errors()
    assert status == ress_gpu.RESS_ERR_BAD_INDEX and detail == 1
    assert ress_gpu.ress_check_device_errors()[0] == 0          # cleared
    qn, kn, vn = np64(q), np64(k), np64(v)
    for i, kept in [(1, [0, 2]), (3, [2, 4]), (0, [0, 2, 4])]:
        ref_o, _ = oracle.sparse_attention_block(qn, kn, vn, kept, 0, i, B)
        assert_attn_close(np64(out)[i * B:(i + 1) * B, 0], ref_o)


def test_float32_inputs_are_staged_and_output_in_float32(ress_gpu, wcache):
    w = workloads.WORKLOADS["tiny"]
    q, k, v = wcache.get(w)
    assert q.dtype == torch.float32
    idx = ress_gpu.ress_select_blocks(q, k, None, w.budget, 0.0, w.block)
    out, lse = _run(ress_gpu, w, q, k, v, idx)
    assert out.dtype == torch.float32


@pytest.mark.parametrize("heads,nb,budget", [(1, 11, 4), (64, 6, 3)])
def test_one_head_and_the_64_head_maximum(heads, nb, budget, ress_gpu):
    B = 64
    g = torch.Generator().manual_seed(heads + nb)
    q, k, v = (torch.randn(nb * B, heads, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    idx = ress_gpu.ress_select_blocks(qd, kd, None, budget, 0.0, B)
    w = workloads.Workload("heads", 1, nb * B, nb * B, heads, 64, "bf16", B, budget, 0.0, 0, "iid")
    out, lse = _run(ress_gpu, w, qd, kd, vd, idx, out_dtype=torch.float32)
    rows = [(h, i) for h in range(heads) for i in range(nb)]
    _compare_rows(q, k, v, idx.cpu().numpy(), out.cpu(), lse.cpu(), B, rows)


def test_grid_near_the_10000_block_limit(ress_gpu):
    """nb = 9,999 key blocks (the kept-block lists of a tile fill most of the
    shared memory): one head, budget 3, sampled rows including the last
    (half-empty) tile."""
    H, nb, B, budget = 1, 9999, 64, 3
    g = torch.Generator().manual_seed(99)
    q, k, v = (torch.randn(nb * B, H, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    rng = np.random.default_rng(99)
    idx = np.sort(np.stack([rng.choice(nb, budget, replace=False) for _ in range(nb)]), -1)
    idx[0] = [0, nb // 2, nb - 1]
    idx = idx.astype(np.int32)[None]
    w = workloads.Workload("wide", 1, nb * B, nb * B, H, 64, "bf16", B, budget, 0.0, 0, "iid")
    out, lse = _run(ress_gpu, w, q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(idx).cuda(),
                    out_dtype=torch.float32)
    rows = [(0, i) for i in (0, 1, 2, 5000, 7777, nb - 2, nb - 1)]
    _compare_rows(q, k, v, idx, out.cpu(), lse.cpu(), B, rows)
    assert torch.isfinite(out).all()
