"""The layout-aware path on the GPU (padding and special tokens) against the
layout oracle: the kept-block masks, the attention outputs and lse of every
row (special queries dense over every valid key, padding queries zero), and
the drift, on a VGGT layout (1,408-token views, 1,374 real, 5 special) with
non-zero padding values, and on a fine layout where some key blocks are
empty and some hold only special tokens.  Outputs start poisoned."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_global_mean_b200 import workloads
from tests.parity import (MASK_MARGIN, assert_attn_close, assert_drift_close, assert_mask_parity,
                          np64, poison, sample_rows)

pytestmark = pytest.mark.gpu


def _vggt_case(views=8, heads=16, seed=11):
    w = workloads.scaled(workloads.WORKLOADS["vggt8"], views, name=f"layout{views}", seed=seed)
    q, k, v = workloads.generate(w)
    # Padding must take part in nothing: give it large random values.
    g = torch.Generator().manual_seed(seed + 1)
    valid, special = oracle.view_layout(w.n_tokens, w.tokens_per_view, w.real_tokens_per_view, 5)
    pad = torch.from_numpy(~valid)
    for x in (q, k, v):
        x[pad] = (8.0 * torch.randn(int(pad.sum()), heads, 64, generator=g)).to(x.dtype)
    layout = (w.tokens_per_view, w.real_tokens_per_view, 5)
    return w, q, k, v, valid, special, layout


def _fine_case(seed=12):
    # Views of 256 tokens, 192 real, the first 64 special, blocks of 64:
    # block 0 of every view is special-only (always kept), block 3 is empty.
    views, t, r, sp, heads, block = 8, 256, 192, 64, 3, 64
    g = torch.Generator().manual_seed(seed)
    n = views * t
    q, k, v = (torch.randn(n, heads, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    valid, special = oracle.view_layout(n, t, r, sp)
    return n, heads, block, q, k, v, valid, special, (t, r, sp)


def _ranked(logits, forced, empty):
    rank = logits.copy()
    rank[:, :, empty] = -np.inf
    rank[:, :, forced] = np.inf
    return rank


def _select(ress, q, k, budget, block, layout):
    n, h = q.shape[0], q.shape[1]
    idx = poison((h, n // block, budget), torch.int32)
    ress.ress_select_blocks_layout(q.cuda(), k.cuda(), budget, block, layout, idx=idx)
    status, detail = ress.ress_check_device_errors()
    assert status == 0, (status, detail)
    return idx


def _attn(ress, q, k, v, idx, block, layout):
    n, h = q.shape[0], q.shape[1]
    out = poison((n, h, 64), torch.float32)
    lse = poison((h, n), torch.float32)
    ress.ress_block_sparse_attn_layout(q.cuda(), k.cuda(), v.cuda(), idx, block, layout, out=out,
                                       lse=lse)
    status, detail = ress.ress_check_device_errors()
    assert status == 0, (status, detail)
    return out, lse


def _compare_attn(q, k, v, idx_np, out, lse, block, valid, special, rows):
    qn, kn, vn = np64(q), np64(k), np64(v)
    o, l = np64(out), np64(lse)
    got_o, ref_o, got_l, ref_l = [], [], [], []
    for h, i in rows:
        ro, rl = oracle.sparse_attention_layout_block(qn, kn, vn, idx_np[h, i], h, i, block,
                                                      valid, special)
        sl = slice(i * block, (i + 1) * block)
        got_o.append(o[sl, h])
        ref_o.append(ro)
        got_l.append(l[h, sl])
        ref_l.append(rl)
    got_o, ref_o = np.concatenate(got_o), np.concatenate(ref_o)
    got_l, ref_l = np.concatenate(got_l), np.concatenate(ref_l)
    pad = np.isneginf(ref_l)
    assert np.array_equal(np.isneginf(got_l), pad), "lse -inf exactly on padding rows"
    assert (got_o[pad] == 0).all(), "padding rows output 0"
    assert_attn_close(got_o, ref_o, got_l[~pad], ref_l[~pad])


def test_vggt_layout_masks_outputs_and_drift_every_row(ress_gpu):
    w, q, k, v, valid, special, layout = _vggt_case()
    nb, H, B = w.n_blocks, w.heads, w.block
    idx = _select(ress_gpu, q, k, w.budget, B, layout)
    ref, sc = oracle.select_blocks_layout(np64(q), np64(k), B, w.budget, valid, special,
                                          return_scores=True)
    assert_mask_parity(idx.cpu().numpy(), ref, _ranked(sc["logits"], sc["forced"], sc["empty"]),
                       w.budget)
    out, lse = _attn(ress_gpu, q, k, v, idx, B, layout)
    idx_np = idx.cpu().numpy()
    rows = [(h, i) for h in range(H) for i in range(nb)]
    _compare_attn(q, k, v, idx_np, out, lse, B, valid, special, rows)
    drift = poison((H, nb, nb - w.budget), torch.float32)
    jset = poison((H, nb), torch.float32)
    ress_gpu.ress_block_drift_layout(q.cuda(), k.cuda(), v.cuda(), idx, lse, B, layout,
                                     drift=drift, set_drift=jset)
    assert ress_gpu.ress_check_device_errors()[0] == 0
    qn, kn, vn, ln = np64(q), np64(k), np64(v), np64(lse)
    ref_d = np.zeros((len(rows[::7]), nb - w.budget))
    ref_j = np.zeros(len(rows[::7]))
    for r, (h, i) in enumerate(rows[::7]):
        ref_d[r], ref_j[r] = oracle.drift_layout_block(qn, kn, vn, idx_np[h, i],
                                                       ln[h, i * B:(i + 1) * B], h, i, B, valid,
                                                       special)
    hs = np.array([h for h, _ in rows[::7]])
    is_ = np.array([i for _, i in rows[::7]])
    assert_drift_close(np64(drift)[hs, is_], ref_d)
    assert_drift_close(np64(jset)[hs, is_], ref_j)


def test_fine_layout_forced_and_empty_blocks(ress_gpu):
    n, H, B, q, k, v, valid, special, layout = _fine_case()
    nb, budget = n // B, 10
    idx = _select(ress_gpu, q, k, budget, B, layout)
    ref, sc = oracle.select_blocks_layout(np64(q), np64(k), B, budget, valid, special,
                                          return_scores=True)
    assert sc["forced"].sum() == 8 and sc["empty"].sum() == 8
    assert_mask_parity(idx.cpu().numpy(), ref, _ranked(sc["logits"], sc["forced"], sc["empty"]),
                       budget, max_excused_frac=0.0)
    got = idx.cpu().numpy()
    forced = np.nonzero(sc["forced"])[0]
    assert all(set(forced.tolist()) <= set(got[h, i].tolist()) for h in range(H) for i in range(nb))
    empty = set(np.nonzero(sc["empty"])[0].tolist())
    assert not any(empty & set(got[h, i].tolist()) for h in range(H) for i in range(nb))
    out, lse = _attn(ress_gpu, q, k, v, idx, B, layout)
    rows = [(h, i) for h in range(H) for i in range(nb)]
    _compare_attn(q, k, v, got, out, lse, B, valid, special, rows)
    drift, jset = ress_gpu.ress_block_drift_layout(q.cuda(), k.cuda(), v.cuda(), idx, lse, B,
                                                   layout)
    assert ress_gpu.ress_check_device_errors()[0] == 0
    qn, kn, vn, ln = np64(q), np64(k), np64(v), np64(lse)
    for h, i in rows[::3]:
        rd, rj = oracle.drift_layout_block(qn, kn, vn, got[h, i], ln[h, i * B:(i + 1) * B], h, i,
                                           B, valid, special)
        assert_drift_close(np64(drift)[h, i], rd)
        assert_drift_close(np64(jset)[h, i:i + 1], np.array([rj]))


def test_a_kept_list_of_empty_blocks_writes_zero_rows(ress_gpu):
    # Rows whose kept blocks hold no valid key: output 0 and lse -inf.
    n, H, B, q, k, v, valid, special, layout = _fine_case(seed=13)
    nb = n // B
    idx = torch.full((H, nb, 1), 3, dtype=torch.int32, device="cuda")     # block 3: empty
    out, lse = _attn(ress_gpu, q, k, v, idx, B, layout)
    o, l = out.cpu(), lse.cpu()
    spec = torch.from_numpy(special)
    assert (o[~spec] == 0).all() and torch.isneginf(l[:, ~spec]).all()
    assert torch.isfinite(l[:, spec]).all()                               # dense rows


def test_views100_layout_sampled_rows(ress_gpu):
    w = workloads.WORKLOADS["views100"]
    q, k, v = workloads.generate(w)
    layout = (w.tokens_per_view, w.real_tokens_per_view, 5)
    valid, special = oracle.view_layout(w.n_tokens, w.tokens_per_view, w.real_tokens_per_view, 5)
    idx = _select(ress_gpu, q, k, w.budget, w.block, layout)
    ref, sc = oracle.select_blocks_layout(np64(q), np64(k), w.block, w.budget, valid, special,
                                          return_scores=True)
    assert_mask_parity(idx.cpu().numpy(), ref, _ranked(sc["logits"], sc["forced"], sc["empty"]),
                       w.budget)
    out, lse = _attn(ress_gpu, q, k, v, idx, w.block, layout)
    rows = sample_rows(w.heads, w.n_blocks, count=24)
    # the first block of view 37 holds special queries
    rows = sorted(set(rows) | {(3, 37 * 22), (9, 99 * 22 + 21)})
    _compare_attn(q, k, v, idx.cpu().numpy(), out, lse, w.block, valid, special, rows)
