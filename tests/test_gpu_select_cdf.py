"""CDF-threshold selection on the GPU against the oracle: counts, kept sets,
padding, truncation to a capacity, the exact-tie and crowded-bin paths, and
the padded list as input of the sparse attention."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_global_mean_b200 import workloads
from tests.parity import MASK_MARGIN, assert_attn_close, np64, poison

pytestmark = pytest.mark.gpu

# The count may differ from float64 only where the cumulative mass is this
# close to tau (float32 probabilities; the GPU's running sum itself is exact).
CDF_MASS_EPS = 1e-5


def _cdf(ress, q, k, tau, block, capacity=None):
    """ress_select_blocks_cdf with poisoned (-1) counts and idx buffers."""
    h, nb = q.shape[1], q.shape[0] // block
    cap = nb if capacity is None else capacity
    return ress.ress_select_blocks_cdf(q, k, tau, block, capacity=capacity,
                                       counts=poison((h, nb), torch.int32, q.device),
                                       idx=poison((h, nb, cap), torch.int32, q.device))


def _check_errors(ress):
    status, detail = ress.ress_check_device_errors()
    assert status == 0, (status, detail)


def _assert_cdf_parity(counts_g, idx_g, probs, logits, tau, cap):
    """counts within the mass tolerance; each row's kept set equals the
    oracle's top min(count, cap) up to the 1e-4 logit margin; padding."""
    h_count, nb, _ = probs.shape
    bad_counts, bad_sets, differ = [], [], 0
    for h in range(h_count):
        for i in range(nb):
            p = probs[h, i]
            order = np.argsort(-p, kind="stable")
            cum = np.cumsum(p[order])
            reached = np.nonzero(cum >= tau)[0]
            k_o = int(reached[0]) + 1 if len(reached) else nb
            k_g = int(counts_g[h, i])
            if k_g != k_o:
                lo, hi = min(k_g, k_o), max(k_g, k_o)
                if not np.all(np.abs(cum[lo - 1:hi - 1] - tau) <= CDF_MASS_EPS):
                    bad_counts.append((h, i, k_g, k_o))
                    continue
            keep = min(k_g, cap)
            row = idx_g[h, i]
            assert (row[keep:] == row[keep - 1]).all(), (h, i)
            got = row[:keep]
            assert np.all(np.diff(got) > 0), (h, i)
            ref = np.sort(order[:keep])
            if set(got.tolist()) != set(ref.tolist()):
                differ += 1
                s = logits[h, i]
                kth = np.sort(s)[::-1][keep - 1]
                for j in set(got.tolist()) ^ set(ref.tolist()):
                    if abs(s[j] - kth) > MASK_MARGIN:
                        bad_sets.append((h, i, j))
                        break
    assert not bad_counts, f"{len(bad_counts)} counts beyond the mass tolerance, e.g. {bad_counts[:5]}"
    assert not bad_sets, f"{len(bad_sets)} kept sets beyond the margin, e.g. {bad_sets[:5]}"
    return differ


@pytest.mark.parametrize("name,tau", [("tiny", 0.5), ("tiny", 0.9), ("vggt8", 0.9),
                                      ("vggt8", 0.98), ("views32", 0.98), ("views100", 0.9),
                                      ("views100", 0.99)])
def test_cdf_selection_matches_oracle(name, tau, ress_gpu, wcache):
    w = workloads.WORKLOADS[name]
    q, k, _ = wcache.get(w)
    tau = float(np.float32(tau))
    counts, idx = _cdf(ress_gpu, q, k, tau, w.block)
    _check_errors(ress_gpu)
    sc = oracle.selection_scores(np64(q), np64(k), None, w.block, 0.0)
    _assert_cdf_parity(counts.cpu().numpy(), idx.cpu().numpy(), sc["probs"], sc["logits"], tau,
                       w.n_blocks)
    again_c, again_i = _cdf(ress_gpu, q, k, tau, w.block)
    assert torch.equal(again_c, counts) and torch.equal(again_i, idx)     # deterministic


def test_cdf_constant_rows_keep_the_lowest_indices(ress_gpu):
    """All-zero queries: every probability is 1/nb, the tie path counts
    ceil(tau nb) blocks and keeps the lowest indices."""
    nb, B, H = 300, 64, 2
    g = torch.Generator().manual_seed(5)
    q = torch.zeros(nb * B, H, 64)
    k = torch.randn(nb * B, H, 64, generator=g)
    tau = float(np.float32(0.4567))
    counts, idx = _cdf(ress_gpu, q.cuda(), k.cuda(), tau, B, capacity=200)
    _check_errors(ress_gpu)
    want = int(np.ceil(tau * nb))
    assert (counts.cpu() == want).all()
    got = idx.cpu().numpy()
    assert (got[:, :, :want] == np.arange(want)[None, None, :]).all()
    assert (got[:, :, want:] == want - 1).all()


def test_cdf_crowded_bin_of_distinct_logits(ress_gpu):
    """Most key blocks have distinct logits packed far closer together than
    one bin of the row's range: the count refines that bin."""
    nb, B = 400, 64
    g = torch.Generator().manual_seed(9)
    u = torch.randn(64, generator=g)
    k = torch.empty(nb * B, 1, 64)
    for j in range(nb):
        if j < 30:   # far below the cluster: almost no probability mass
            kb = -2.0 * u + 0.5 * torch.randn(64, generator=g)
        else:        # the cluster: 97 distinct logits 1e-3 apart (repeated blocks tie)
            kb = u + 1e-3 * (j % 97) * torch.ones(64)
        k[j * B:(j + 1) * B, 0] = kb
    q = (u + 0.1 * torch.randn(nb * B, 1, 64, generator=g)).float()
    sc = oracle.selection_scores(np64(q), np64(k), None, B, 0.0)
    for tau in (0.3, 0.7, 0.95):
        tau = float(np.float32(tau))
        counts, idx = _cdf(ress_gpu, q.cuda(), k.cuda(), tau, B)
        _check_errors(ress_gpu)
        _assert_cdf_parity(counts.cpu().numpy(), idx.cpu().numpy(), sc["probs"], sc["logits"],
                           tau, nb)


def test_cdf_truncates_to_the_capacity_and_feeds_attention(ress_gpu, wcache):
    w = workloads.WORKLOADS["vggt8"]
    q, k, v = wcache.get(w)
    tau, cap = float(np.float32(0.95)), 40
    counts, idx = _cdf(ress_gpu, q, k, tau, w.block, capacity=cap)
    _check_errors(ress_gpu)
    sc = oracle.selection_scores(np64(q), np64(k), None, w.block, 0.0)
    _assert_cdf_parity(counts.cpu().numpy(), idx.cpu().numpy(), sc["probs"], sc["logits"], tau, cap)
    assert (counts.cpu() > cap).any()        # some rows are truncated to their top 40
    # The padded list is a valid fixed-capacity input of the sparse attention.
    out, lse = ress_gpu.ress_block_sparse_attn(q, k, v, idx, w.block, out_dtype=torch.float32)
    _check_errors(ress_gpu)
    idx_np = idx.cpu().numpy()
    rows = [(0, 0), (3, 17), (15, w.n_blocks - 1)]
    for h, i in rows:
        kept = sorted(set(idx_np[h, i].tolist()))
        o_ref, l_ref = oracle.sparse_attention_block(np64(q), np64(k), np64(v), kept, h, i, w.block)
        o = out[i * w.block:(i + 1) * w.block, h].double().cpu().numpy()
        assert_attn_close(o, o_ref)
