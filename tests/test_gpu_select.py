"""Stage 1 on the GPU against the oracle: pooled means, full kept-block masks
at every workload size, and the lowest-index tie rule."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_global_mean_b200 import workloads
from tests.parity import assert_mask_parity, np64

pytestmark = pytest.mark.gpu

ALL = ["tiny", "vggt8", "views32", "views100", "views200"]


def _check_errors(ress):
    status, detail = ress.ress_check_device_errors()
    assert status == 0, (status, detail)


@pytest.mark.parametrize("name", ["tiny", "vggt8", "views32"])
def test_pooled_means_match_oracle(name, ress_gpu, wcache):
    w = workloads.WORKLOADS[name]
    q, k, v = wcache.get(w)
    nb, H = w.n_blocks, w.heads
    need = ress_gpu.select_workspace_bytes(w.n_tokens, H, w.block, q.dtype, w.lam)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ress_gpu.ress_select_blocks(q, k, v if w.lam else None, w.budget, w.lam, w.block, workspace=ws)
    _check_errors(ress_gpu)
    fl = ws.view(torch.float32)
    nb_pad = (nb + 255) // 256 * 256
    qbar = fl[:H * nb * 64].view(H, nb, 64)
    off = (H * nb * 64 * 4 + 255) // 256 * 256 // 4
    kbar_t = fl[off:off + H * 64 * nb_pad].view(H, 64, nb_pad)[:, :, :nb]
    np.testing.assert_allclose(np64(qbar), oracle.pool_blocks(np64(q), w.block), rtol=2e-6, atol=2e-6)
    np.testing.assert_allclose(np64(kbar_t).transpose(0, 2, 1), oracle.pool_blocks(np64(k), w.block),
                               rtol=2e-6, atol=2e-6)


@pytest.mark.parametrize("name", ALL)
def test_full_mask_matches_oracle(name, ress_gpu, wcache):
    w = workloads.WORKLOADS[name]
    q, k, v = wcache.get(w)
    idx = ress_gpu.ress_select_blocks(q, k, v if w.lam else None, w.budget, w.lam, w.block)
    _check_errors(ress_gpu)
    ref, sc = oracle.select_blocks(np64(q), np64(k), np64(v) if w.lam else None, w.block,
                                   w.budget, w.lam, return_scores=True)
    ranked = sc["logits"] if w.lam == 0 else sc["score"]
    assert_mask_parity(idx.cpu().numpy(), ref, ranked, w.budget)


def test_selection_is_deterministic(ress_gpu, wcache):
    w = workloads.WORKLOADS["vggt8"]
    q, k, v = wcache.get(w)
    a = ress_gpu.ress_select_blocks(q, k, None, w.budget, 0.0, w.block)
    b = ress_gpu.ress_select_blocks(q, k, None, w.budget, 0.0, w.block)
    assert torch.equal(a, b)


@pytest.mark.parametrize("block", [64, 128])
def test_duplicated_key_block_keeps_the_lower_index(block, ress_gpu):
    g = torch.Generator().manual_seed(5)
    nb, H = 12, 2
    q = torch.randn(nb * block, H, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(nb * block, H, 64, generator=g).to(torch.bfloat16)
    k[9 * block:10 * block] = k[3 * block:4 * block]          # block 9 is a copy of block 3
    qd, kd = q.cuda(), k.cuda()
    ref, sc = oracle.select_blocks(np64(q), np64(k), None, block, 1, 0.0, return_scores=True)
    for h in range(H):
        for i in range(nb):
            row = sc["logits"][h, i]
            assert row[3] == row[9]
            budget = int(np.nonzero(np.argsort(-row, kind="stable") == 3)[0][0]) + 1
            idx = ress_gpu.ress_select_blocks(qd, kd, None, budget, 0.0, block).cpu().numpy()
            assert 3 in idx[h, i] and 9 not in idx[h, i]
    _check_errors(ress_gpu)


@pytest.mark.parametrize("budget", [1, 2, 7, 8])
def test_budget_extremes_on_odd_block_count(budget, ress_gpu):
    g = torch.Generator().manual_seed(budget)
    nb, H, B = 8, 3, 64
    q = torch.randn(nb * B, H, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(nb * B, H, 64, generator=g).to(torch.bfloat16)
    idx = ress_gpu.ress_select_blocks(q.cuda(), k.cuda(), None, budget, 0.0, B)
    _check_errors(ress_gpu)
    ref, sc = oracle.select_blocks(np64(q), np64(k), None, B, budget, 0.0, return_scores=True)
    assert_mask_parity(idx.cpu().numpy(), ref, sc["logits"], budget, max_excused_frac=0.0)


def _random_case(nb, heads, block, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(nb * block, heads, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(nb * block, heads, 64, generator=g).to(torch.bfloat16)
    return q, k


@pytest.mark.parametrize("nb,budget", [(13, 5), (2533, 253), (4096, 409)])
def test_row_lengths_and_both_tile_shapes(nb, budget, ress_gpu):
    """Odd row lengths (a ragged last run per lane), the eight-row CTA used
    above 2,532 blocks, and the largest supported grid (4,096 blocks)."""
    q, k = _random_case(nb, 1, 64, seed=nb)
    idx = ress_gpu.ress_select_blocks(q.cuda(), k.cuda(), None, budget, 0.0, 64)
    _check_errors(ress_gpu)
    ref, sc = oracle.select_blocks(np64(q), np64(k), None, 64, budget, 0.0, return_scores=True)
    assert_mask_parity(idx.cpu().numpy(), ref, sc["logits"], budget)


def test_crowded_threshold_bin_and_constant_rows(ress_gpu):
    """Many bitwise-equal pooled scores around the budget-th value (the
    threshold bin holds far more than the exactly ranked candidates), and
    all-zero queries whose rows are constant: the lowest indices win."""
    nb, B, budget = 300, 64, 100
    g = torch.Generator().manual_seed(7)
    k = torch.randn(nb * B, 2, 64, generator=g)
    k[40 * B:] = k[:B].repeat(nb - 40, 1, 1)                 # blocks 40.. copy block 0
    q = torch.randn(nb * B, 2, 64, generator=g)
    q[:, 1] = 0.0                                            # head 1: every score is 0
    q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    idx = ress_gpu.ress_select_blocks(q.cuda(), k.cuda(), None, budget, 0.0, B).cpu().numpy()
    _check_errors(ress_gpu)
    ref, sc = oracle.select_blocks(np64(q), np64(k), None, B, budget, 0.0, return_scores=True)
    assert_mask_parity(idx, ref, sc["logits"], budget, max_excused_frac=0.0)
    assert (idx[1] == np.arange(budget)[None, :]).all()
