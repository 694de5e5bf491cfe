"""Stage 1 on the GPU against the oracle: pooled means (Q, K and V) and the
value contrast element by element, full kept-block masks at every workload
size, head counts from 1 to 64, and the lowest-index tie rule.  Every output
buffer starts poisoned (-1), so a row the kernel skips cannot pass."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_global_mean_b200 import workloads
from tests.parity import assert_mask_parity, np64, poison

pytestmark = pytest.mark.gpu

ALL = ["tiny", "vggt8", "views32", "views100", "views200"]


def _check_errors(ress):
    status, detail = ress.ress_check_device_errors()
    assert status == 0, (status, detail)


def _select(ress, q, k, v, budget, lam, block, **kw):
    n, h = q.shape[0], q.shape[1]
    idx = poison((h, n // block, budget), torch.int32, q.device)
    return ress.ress_select_blocks(q, k, v, budget, lam, block, idx=idx, **kw)


def _workspace_views(ws, H, nb, with_v, tc):
    """Qbar [H][nb][64] and the pooled keys as [H][nb][64] (from Kbar^T, or
    from the tf32 high + low planes of the tensor-core layout), Vbar and the
    contrast: the layouts include/ress.h gives for the selection workspace."""
    fl = ws.view(torch.float32)
    nb_pad = (nb + 255) // 256 * 256

    def up(nbytes):
        return (nbytes + 255) // 256 * 256 // 4

    off = 0
    qbar = fl[off:off + H * nb * 64].view(H, nb, 64)
    off += up(H * nb * 64 * 4)
    if tc:
        plane = up(H * nb_pad * 64 * 4)
        khi = fl[off:off + H * nb_pad * 64].view(H, nb_pad, 64)[:, :nb]
        klo = fl[off + plane:off + plane + H * nb_pad * 64].view(H, nb_pad, 64)[:, :nb]
        return qbar, khi.double() + klo.double(), None, None
    kbar = fl[off:off + H * 64 * nb_pad].view(H, 64, nb_pad)[:, :, :nb].transpose(1, 2)
    off += up(H * 64 * nb_pad * 4)
    vbar = contrast = None
    if with_v:
        vbar = fl[off:off + H * nb * 64].view(H, nb, 64)
        off += up(H * nb * 64 * 4)
        contrast = fl[off:off + H * nb].view(H, nb)
    return qbar, kbar, vbar, contrast


@pytest.mark.parametrize("name", ["tiny", "vggt8", "views32"])
def test_pooled_means_and_contrast_match_oracle(name, ress_gpu, wcache):
    w = workloads.WORKLOADS[name]
    q, k, v = wcache.get(w)
    nb, H = w.n_blocks, w.heads
    need = ress_gpu.select_workspace_bytes(w.n_tokens, H, w.block, q.dtype, w.lam)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")   # NaN-filled floats
    _select(ress_gpu, q, k, v if w.lam else None, w.budget, w.lam, w.block, workspace=ws)
    _check_errors(ress_gpu)
    tc = w.lam == 0 and w.budget < nb <= 2304          # the tensor-core selection's layout
    qbar, kbar, vbar, contrast = _workspace_views(ws, H, nb, bool(w.lam), tc)
    np.testing.assert_allclose(np64(qbar), oracle.pool_blocks(np64(q), w.block), rtol=2e-6, atol=2e-6)
    # tf32 high + low parts hold a float32 value to about 2^-22 relative
    np.testing.assert_allclose(np64(kbar), oracle.pool_blocks(np64(k), w.block),
                               rtol=2e-6 if not tc else 4e-6, atol=2e-6)
    if w.lam:
        ref_vbar = oracle.pool_blocks(np64(v), w.block)
        np.testing.assert_allclose(np64(vbar), ref_vbar, rtol=2e-6, atol=2e-6)
        # The contrast of the GPU's own pooled values (float32 differences).
        np.testing.assert_allclose(np64(contrast), oracle.value_contrast(ref_vbar),
                                   rtol=1e-5, atol=1e-5)
        assert (contrast[:, 0] == 0).all()


@pytest.mark.parametrize("name", ALL)
def test_full_mask_matches_oracle(name, ress_gpu, wcache):
    w = workloads.WORKLOADS[name]
    q, k, v = wcache.get(w)
    idx = _select(ress_gpu, q, k, v if w.lam else None, w.budget, w.lam, w.block)
    _check_errors(ress_gpu)
    ref, sc = oracle.select_blocks(np64(q), np64(k), np64(v) if w.lam else None, w.block,
                                   w.budget, w.lam, return_scores=True)
    ranked = sc["logits"] if w.lam == 0 else sc["score"]
    assert_mask_parity(idx.cpu().numpy(), ref, ranked, w.budget)


def test_selection_is_deterministic(ress_gpu, wcache):
    w = workloads.WORKLOADS["vggt8"]
    q, k, v = wcache.get(w)
    a = _select(ress_gpu, q, k, None, w.budget, 0.0, w.block)
    b = _select(ress_gpu, q, k, None, w.budget, 0.0, w.block)
    assert torch.equal(a, b)


@pytest.mark.parametrize("heads,nb,budget,lam", [(1, 37, 9, 0.0), (1, 21, 5, 0.5),
                                                 (64, 12, 5, 0.0), (64, 9, 4, 0.5)])
def test_one_head_and_the_64_head_maximum(heads, nb, budget, lam, ress_gpu):
    g = torch.Generator().manual_seed(heads * 100 + nb)
    q, k, v = (torch.randn(nb * 64, heads, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    idx = _select(ress_gpu, q.cuda(), k.cuda(), v.cuda() if lam else None, budget, lam, 64)
    _check_errors(ress_gpu)
    ref, sc = oracle.select_blocks(np64(q), np64(k), np64(v) if lam else None, 64, budget, lam,
                                   return_scores=True)
    ranked = sc["logits"] if lam == 0 else sc["score"]
    assert_mask_parity(idx.cpu().numpy(), ref, ranked, budget)


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
            idx = _select(ress_gpu, qd, kd, None, budget, 0.0, block).cpu().numpy()
            assert 3 in idx[h, i] and 9 not in idx[h, i]
    _check_errors(ress_gpu)


@pytest.mark.parametrize("budget", [1, 2, 7, 8])
def test_budget_extremes_on_odd_block_count(budget, ress_gpu):
    g = torch.Generator().manual_seed(budget)
    nb, H, B = 8, 3, 64
    q = torch.randn(nb * B, H, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(nb * B, H, 64, generator=g).to(torch.bfloat16)
    idx = _select(ress_gpu, q.cuda(), k.cuda(), None, budget, 0.0, B)
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
    idx = _select(ress_gpu, q.cuda(), k.cuda(), None, budget, 0.0, 64)
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
    idx = _select(ress_gpu, q.cuda(), k.cuda(), None, budget, 0.0, B).cpu().numpy()
    _check_errors(ress_gpu)
    ref, sc = oracle.select_blocks(np64(q), np64(k), None, B, budget, 0.0, return_scores=True)
    assert_mask_parity(idx, ref, sc["logits"], budget, max_excused_frac=0.0)
    assert (idx[1] == np.arange(budget)[None, :]).all()
