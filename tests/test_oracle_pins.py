"""Pins of the CPU oracle against facts that do not come from the oracle itself:
closed forms, a hand-worked example, brute force on tiny inputs, invariants and
independent library routines (torch float64 on the CPU).

Each test is chosen so that a plausible slip in the oracle (sum instead of
mean, sqrt(B) instead of sqrt(d), j+1 instead of j-1, ties to the higher index,
a causal or missing mask, the dense instead of the kept-set normaliser, a norm
other than Frobenius) fails at least one of them.
"""

import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from block_sparse_global_mean_b200 import workloads


def _np64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def _tiny_inputs():
    w = workloads.WORKLOADS["tiny"]
    q, k, v = workloads.generate(w)
    return w, _np64(q), _np64(k), _np64(v)


# --------------------------------------------------------------------------
# Pooling
# --------------------------------------------------------------------------

def test_pool_constant_blocks_pool_to_the_constant():
    rng = np.random.default_rng(11)
    B, nb, H, d = 16, 5, 3, 8
    const = rng.integers(-64, 64, size=(nb, H, d)) / 8.0  # dyadic: sums are exact
    x = np.repeat(const, B, axis=0)                       # every block constant
    got = oracle.pool_blocks(x, B)
    np.testing.assert_array_equal(got, const.transpose(1, 0, 2))


def test_pool_is_invariant_to_token_order_inside_a_block():
    rng = np.random.default_rng(12)
    B, nb, H, d = 16, 6, 2, 8
    x = rng.normal(size=(nb * B, H, d))
    perm = np.concatenate([i * B + rng.permutation(B) for i in range(nb)])
    np.testing.assert_allclose(oracle.pool_blocks(x[perm], B), oracle.pool_blocks(x, B),
                               rtol=0, atol=1e-14)


def test_pool_matches_torch_mean_over_contiguous_blocks():
    rng = np.random.default_rng(13)
    B, nb, H, d = 32, 7, 4, 64
    x = rng.normal(size=(nb * B, H, d))
    ref = torch.from_numpy(x).view(nb, B, H, d).mean(dim=1).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(oracle.pool_blocks(x, B), ref, rtol=1e-13, atol=1e-14)


# --------------------------------------------------------------------------
# Pooled scores
# --------------------------------------------------------------------------

def test_logit_temperature_is_sqrt_head_dim_not_sqrt_block():
    d = 64
    qbar = np.zeros((1, 1, d))
    kbar = np.zeros((1, 2, d))
    qbar[0, 0, 0] = 2.0
    kbar[0, 0, 0] = 3.0       # dot = 6
    kbar[0, 1, 1] = 5.0       # dot = 0
    s = oracle.block_logits(qbar, kbar)
    assert s[0, 0, 0] == pytest.approx(6.0 / 8.0, abs=1e-15)
    assert s[0, 0, 1] == 0.0


def test_probs_rows_sum_to_one_and_match_torch_softmax():
    w, q, k, v = _tiny_inputs()
    sc = oracle.selection_scores(q, k, v, w.block, 0.0)
    np.testing.assert_allclose(sc["probs"].sum(-1), 1.0, rtol=0, atol=1e-12)
    tq = torch.from_numpy(q).view(w.n_blocks, w.block, w.heads, 64).mean(1).permute(1, 0, 2)
    tk = torch.from_numpy(k).view(w.n_blocks, w.block, w.heads, 64).mean(1).permute(1, 0, 2)
    ref = torch.softmax(tq @ tk.transpose(1, 2) / 8.0, dim=-1).numpy()
    np.testing.assert_allclose(sc["probs"], ref, rtol=1e-12, atol=1e-15)


def test_lambda_zero_ranking_by_probability_equals_ranking_by_logit():
    w, q, k, v = _tiny_inputs()
    sc = oracle.selection_scores(q, k, v, w.block, 0.0)
    np.testing.assert_array_equal(oracle.topk_lowest_index(sc["probs"], w.budget),
                                  oracle.topk_lowest_index(sc["logits"], w.budget))


def test_value_contrast_closed_form_uses_previous_block():
    H, nb, d = 2, 9, 64
    vbar = np.zeros((H, nb, d))
    for j in range(nb):
        vbar[:, j, 0] = j * j                # ||Vbar_j - Vbar_{j-1}|| = 2j - 1
    c = oracle.value_contrast(vbar)
    expect = np.array([0.0] + [2.0 * j - 1.0 for j in range(1, nb)])
    np.testing.assert_allclose(c, np.broadcast_to(expect, (H, nb)), rtol=0, atol=1e-12)


def test_value_contrast_of_constant_values_is_zero_and_lambda_zero_reduces():
    rng = np.random.default_rng(14)
    B, nb, H, d = 16, 6, 2, 64
    q = rng.normal(size=(nb * B, H, d))
    k = rng.normal(size=(nb * B, H, d))
    v = np.broadcast_to(rng.normal(size=(1, H, d)), (nb * B, H, d)).copy()
    sc = oracle.selection_scores(q, k, v, B, 0.7)
    np.testing.assert_allclose(sc["contrast"], 0.0, atol=1e-14)
    np.testing.assert_allclose(sc["score"], sc["probs"], atol=1e-14)


def test_contrast_enters_the_score_additively_with_weight_lambda():
    rng = np.random.default_rng(15)
    B, nb, H, d = 16, 6, 2, 64
    q, k, v = (rng.normal(size=(nb * B, H, d)) for _ in range(3))
    lam = 0.37
    sc = oracle.selection_scores(q, k, v, B, lam)
    vb = torch.from_numpy(v).view(nb, B, H, d).mean(1).permute(1, 0, 2)
    c = torch.zeros(H, nb, dtype=torch.float64)
    c[:, 1:] = torch.linalg.vector_norm(vb[:, 1:] - vb[:, :-1], dim=-1)
    np.testing.assert_allclose(sc["score"] - sc["probs"],
                               np.broadcast_to(lam * c.numpy()[:, None, :], sc["score"].shape),
                               rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------
# Top-k
# --------------------------------------------------------------------------

def _brute_force_topk(row, k):
    """Subset maximising the score sum; ties to the lexicographically smallest
    ascending index tuple."""
    best, best_sum = None, -math.inf
    for comb in itertools.combinations(range(len(row)), k):   # ascending tuples, lexicographic
        s = float(sum(row[j] for j in comb))
        if s > best_sum:
            best, best_sum = comb, s
    return list(best)


def test_topk_equals_brute_force_on_tiny():
    w, q, k, v = _tiny_inputs()
    idx, sc = oracle.select_blocks(q, k, v, w.block, w.budget, 0.0, return_scores=True)
    assert idx.shape == (w.heads, w.n_blocks, w.budget)
    for h in range(w.heads):
        for i in range(w.n_blocks):
            assert list(idx[h, i]) == _brute_force_topk(sc["score"][h, i], w.budget)


def test_topk_with_many_ties_matches_brute_force():
    rng = np.random.default_rng(16)
    for _ in range(40):
        row = rng.integers(0, 3, size=8).astype(np.float64)     # heavy ties
        for kk in (1, 3, 4, 7):
            got = oracle.topk_lowest_index(row[None, None, :], kk)[0, 0]
            assert list(got) == _brute_force_topk(row, kk)


def test_cdf_threshold_closed_forms_on_dyadic_rows():
    # Exact dyadic probabilities: every partial sum is exact, so "reaches"
    # (>=) and "exceeds" (>) differ visibly when tau equals a partial sum.
    row = np.array([0.125, 0.5, 0.0625, 0.25, 0.0625])[None, None, :]
    assert oracle.cdf_counts(row, 0.5)[0, 0] == 1       # the largest alone reaches 0.5
    assert oracle.cdf_counts(row, 0.75)[0, 0] == 2      # 0.5 + 0.25
    assert oracle.cdf_counts(row, 0.7500001)[0, 0] == 3
    assert oracle.cdf_counts(row, 0.1)[0, 0] == 1       # tau below the maximum
    assert oracle.cdf_counts(row, 1.0)[0, 0] == 5       # the whole row
    assert oracle.cdf_counts(row, 2.0)[0, 0] == 5       # never reached: every block


def test_cdf_threshold_on_uniform_rows_is_ceil_tau_nb():
    for nb in (7, 8, 50):
        row = np.full((1, 1, nb), 1.0 / nb)
        for tau in (0.13, 0.5, 0.61, 0.97):
            assert oracle.cdf_counts(row, tau)[0, 0] == math.ceil(tau * nb - 1e-9)


def _brute_force_cdf(row, tau):
    """Smallest subset reaching mass tau; among those, the largest mass, then
    the lexicographically smallest ascending tuple."""
    n = len(row)
    for m in range(1, n + 1):
        best, best_sum = None, -1.0
        for comb in itertools.combinations(range(n), m):
            s = float(sum(row[j] for j in comb))
            if s >= tau and s > best_sum:
                best, best_sum = comb, s
        if best is not None:
            return m, list(best)
    return n, list(range(n))


def test_cdf_selection_equals_brute_force_on_tiny():
    w, q, k, v = _tiny_inputs()
    for tau in (0.3, 0.55, 0.8, 0.95):
        counts, idx, sc = oracle.select_blocks_cdf(q, k, w.block, tau, w.n_blocks,
                                                   return_scores=True)
        assert idx.shape == (w.heads, w.n_blocks, w.n_blocks)
        for h in range(w.heads):
            for i in range(w.n_blocks):
                m, kept = _brute_force_cdf(sc["probs"][h, i], tau)
                assert counts[h, i] == m
                assert list(idx[h, i, :m]) == kept
                assert (idx[h, i, m:] == kept[-1]).all()


def test_cdf_counts_grow_with_tau_and_capacity_truncates_to_the_top_blocks():
    w, q, k, v = _tiny_inputs()
    probs = oracle.selection_scores(q, k, None, w.block, 0.0)["probs"]
    prev = np.zeros(probs.shape[:2], dtype=np.int32)
    for tau in np.linspace(0.05, 1.0, 20):
        c = oracle.cdf_counts(probs, float(tau))
        assert (c >= prev).all() and (c >= 1).all() and (c <= w.n_blocks).all()
        prev = c
    for tau in (0.3, 0.99):
        counts, idx = oracle.select_blocks_cdf(q, k, w.block, tau, 2)
        for h in range(w.heads):
            for i in range(w.n_blocks):
                keep = min(2, int(counts[h, i]))
                kept = sorted(np.argsort(-probs[h, i], kind="stable")[:keep].tolist())
                assert list(idx[h, i]) == kept + [kept[-1]] * (2 - keep)


def test_topk_duplicated_key_block_keeps_lower_index():
    # Block 6 is a copy of block 2, so their pooled scores are bitwise equal.
    rng = np.random.default_rng(17)
    B, nb, H, d = 64, 8, 1, 64
    q = rng.normal(size=(nb * B, H, d))
    k = rng.normal(size=(nb * B, H, d))
    k[6 * B:7 * B] = k[2 * B:3 * B]
    sc = oracle.selection_scores(q, k, None, B, 0.0)
    for i in range(nb):
        s = sc["score"][0, i]
        assert s[2] == s[6]
        order = np.argsort(-s, kind="stable")
        pos = int(np.nonzero(order == 2)[0][0])
        kk = pos + 1                  # the boundary falls between the twins
        got = oracle.topk_lowest_index(sc["score"][:, i:i + 1], kk)[0, 0]
        assert 2 in got and 6 not in got


# --------------------------------------------------------------------------
# Sparse attention
# --------------------------------------------------------------------------

def _sdpa(q, k, v, mask=None):
    """torch SDPA in float64 on the CPU for one head: q [Nq, d], k/v [Nk, d]."""
    tq = torch.from_numpy(q)[None, None]
    tk = torch.from_numpy(k)[None, None]
    tv = torch.from_numpy(v)[None, None]
    am = None if mask is None else torch.from_numpy(mask)[None, None]
    return F.scaled_dot_product_attention(tq, tk, tv, attn_mask=am)[0, 0].numpy()


def test_full_budget_reproduces_dense_attention():
    w, q, k, v = _tiny_inputs()
    nb = w.n_blocks
    idx = np.tile(np.arange(nb, dtype=np.int32), (w.heads, nb, 1))
    out, lse = oracle.sparse_attention(q, k, v, idx, w.block)
    for h in range(w.heads):
        ref = _sdpa(q[:, h], k[:, h], v[:, h])
        np.testing.assert_allclose(out[:, h], ref, rtol=1e-10, atol=1e-12)
        ref_lse = torch.logsumexp(torch.from_numpy(q[:, h] @ k[:, h].T / 8.0), dim=-1).numpy()
        np.testing.assert_allclose(lse[h], ref_lse, rtol=1e-12, atol=1e-12)


def test_sparse_attention_equals_dense_with_minus_inf_mask():
    w, q, k, v = _tiny_inputs()
    rng = np.random.default_rng(18)
    nb, B = w.n_blocks, w.block
    idx = np.sort(np.stack([np.stack([rng.choice(nb, w.budget, replace=False)
                                      for _ in range(nb)]) for _ in range(w.heads)]), -1)
    idx = idx.astype(np.int32)
    out, lse = oracle.sparse_attention(q, k, v, idx, B)
    for h in range(w.heads):
        mask = np.full((w.n_tokens, w.n_tokens), -np.inf)
        for i in range(nb):
            for j in idx[h, i]:
                mask[i * B:(i + 1) * B, j * B:(j + 1) * B] = 0.0
        ref = _sdpa(q[:, h], k[:, h], v[:, h], mask)
        np.testing.assert_allclose(out[:, h], ref, rtol=1e-10, atol=1e-12)
        logits = torch.from_numpy(q[:, h] @ k[:, h].T / 8.0 + mask)
        np.testing.assert_allclose(lse[h], torch.logsumexp(logits, -1).numpy(), rtol=1e-12)


def test_dropping_the_max_score_block_changes_the_output():
    w, q, k, v = _tiny_inputs()
    idx, sc = oracle.select_blocks(q, k, v, w.block, w.budget, 0.0, return_scores=True)
    nb = w.n_blocks
    for h in range(w.heads):
        for i in range(nb):
            row = sc["score"][h, i]
            top = int(np.argmax(row))
            alt = [j for j in np.argsort(-row, kind="stable") if j != top][:w.budget]
            o1, _ = oracle.sparse_attention_block(q, k, v, idx[h, i], h, i, w.block)
            o2, _ = oracle.sparse_attention_block(q, k, v, sorted(alt), h, i, w.block)
            assert np.abs(o1 - o2).max() >= 1e-3


# --------------------------------------------------------------------------
# Hand-worked example through all three stages (d = 4, B = 2, N = 4, k = 1)
# --------------------------------------------------------------------------

def _hand_inputs():
    q = np.zeros((4, 1, 4)); k = np.zeros((4, 1, 4)); v = np.zeros((4, 1, 4))
    q[0, 0, 0] = 2.0          # Qbar_0 = (1, 0, 0, 0)
    q[2, 0, 1] = 2.0          # Qbar_1 = (0, 1, 0, 0)
    k[0, 0, 0] = 4.0          # Kbar_0 = (2, 0, 0, 0)
    k[3, 0, 1] = 6.0          # Kbar_1 = (0, 3, 0, 0)
    for t in range(4):
        v[t, 0, t] = 1.0      # V_t = e_t
    return q, k, v


def test_hand_worked_example():
    q, k, v = _hand_inputs()
    e = math.e
    sc = oracle.selection_scores(q, k, v, 2, 0.0)
    # logits = Qbar Kbar^T / sqrt(4): [[1, 0], [0, 1.5]]
    np.testing.assert_allclose(sc["logits"][0], [[1.0, 0.0], [0.0, 1.5]], atol=1e-15)
    np.testing.assert_allclose(sc["probs"][0], [[e / (e + 1), 1 / (e + 1)],
                                                [1 / (1 + e ** 1.5), e ** 1.5 / (1 + e ** 1.5)]],
                               rtol=1e-14)
    idx = oracle.topk_lowest_index(sc["score"], 1)
    assert idx[0, :, 0].tolist() == [0, 1]
    out, lse = oracle.sparse_attention(q, k, v, idx, 2)
    # token 0: logits (4, 0) over keys 0, 1; token 1: (0, 0); token 2: (0, 6) over keys 2, 3.
    expect = np.array([[e ** 4 / (1 + e ** 4), 1 / (1 + e ** 4), 0, 0],
                       [0.5, 0.5, 0, 0],
                       [0, 0, 1 / (1 + e ** 6), e ** 6 / (1 + e ** 6)],
                       [0, 0, 0.5, 0.5]])
    np.testing.assert_allclose(out[:, 0], expect, rtol=1e-14, atol=1e-16)
    np.testing.assert_allclose(lse[0], [math.log(1 + e ** 4), math.log(2),
                                        math.log(1 + e ** 6), math.log(2)], rtol=1e-14)
    drift, jset = oracle.block_drift(q, k, v, idx, lse, 2)
    # Query block 0 drops block 1: all four logits are 0, so
    # C = [[0, 0, 1, 1] / (1 + e^4), [0, 0, 1, 1] / 2].
    d0 = math.sqrt(2.0 / (1 + e ** 4) ** 2 + 2.0 / 4.0)
    # Query block 1 drops block 0: C = [[1, 1, 0, 0] / (1 + e^6), [1, 1, 0, 0] / 2].
    d1 = math.sqrt(2.0 / (1 + e ** 6) ** 2 + 2.0 / 4.0)
    np.testing.assert_allclose(drift[0, :, 0], [d0, d1], rtol=1e-14)
    np.testing.assert_allclose(jset[0], [d0, d1], rtol=1e-14)


# --------------------------------------------------------------------------
# Drift
# --------------------------------------------------------------------------

def test_drift_of_an_empty_drop_set_is_zero():
    w, q, k, v = _tiny_inputs()
    nb = w.n_blocks
    idx = np.tile(np.arange(nb, dtype=np.int32), (w.heads, nb, 1))
    _, lse = oracle.sparse_attention(q, k, v, idx, w.block)
    drift, jset = oracle.block_drift(q, k, v, idx, lse, w.block)
    assert drift.shape == (w.heads, nb, 0)
    np.testing.assert_array_equal(jset, 0.0)


def test_drift_reconstructs_dense_attention():
    """O_dense = (O_sparse + sum_j C_j) / (1 + sum_j r_j), r_j = sum_t exp(s - lse).

    The expected J = ||sum_j C_j||_F is formed from torch SDPA and torch
    logsumexp only, then compared with the oracle's J.
    """
    w, q, k, v = _tiny_inputs()
    idx = oracle.select_blocks(q, k, v, w.block, w.budget)
    _, lse = oracle.sparse_attention(q, k, v, idx, w.block)
    _, jset = oracle.block_drift(q, k, v, idx, lse, w.block)
    B, nb = w.block, w.n_blocks
    for h in range(w.heads):
        logits = q[:, h] @ k[:, h].T / 8.0
        dense = _sdpa(q[:, h], k[:, h], v[:, h])
        for i in range(nb):
            keep = np.full(w.n_tokens, False)
            for j in idx[h, i]:
                keep[j * B:(j + 1) * B] = True
            rows = slice(i * B, (i + 1) * B)
            mask = np.where(keep, 0.0, -np.inf)[None, :].repeat(B, 0)
            sparse = _sdpa(q[rows, h], k[:, h], v[:, h], mask)
            lse_t = torch.logsumexp(torch.from_numpy(logits[rows] + mask), -1).numpy()
            r = np.exp(logits[rows][:, ~keep] - lse_t[:, None]).sum(-1)
            total_c = dense[rows] * (1.0 + r[:, None]) - sparse
            assert jset[h, i] == pytest.approx(np.linalg.norm(total_c), rel=1e-9)


def test_drift_of_one_dropped_block_equals_j_and_triangle_inequality_holds():
    w, q, k, v = _tiny_inputs()
    nb = w.n_blocks
    rng = np.random.default_rng(19)
    idx1 = np.stack([np.stack([np.sort(rng.choice(nb, nb - 1, replace=False))
                               for _ in range(nb)]) for _ in range(w.heads)]).astype(np.int32)
    _, lse1 = oracle.sparse_attention(q, k, v, idx1, w.block)
    drift1, j1 = oracle.block_drift(q, k, v, idx1, lse1, w.block)
    np.testing.assert_allclose(drift1[..., 0], j1, rtol=1e-14)
    idx = oracle.select_blocks(q, k, v, w.block, w.budget)
    _, lse = oracle.sparse_attention(q, k, v, idx, w.block)
    drift, jset = oracle.block_drift(q, k, v, idx, lse, w.block)
    assert np.all(jset <= drift.sum(-1) * (1 + 1e-12))
    assert np.all(jset < drift.sum(-1))   # generic contributions are not parallel


def test_drift_closed_form_with_zero_queries_and_orthogonal_values():
    """Q = 0 makes every logit 0, so exp(s - lse) = 1 / (k B) for all tokens and
    C_j[n] = sum_{t in j} V[t] / (k B) for every query row.  Values of dropped
    block j live on coordinate j only, so the C_j are orthogonal and
    J^2 = sum_j drift_j^2."""
    B, nb, H, d, budget = 8, 6, 1, 16, 2
    rng = np.random.default_rng(20)
    q = np.zeros((nb * B, H, d))
    k = rng.normal(size=(nb * B, H, d))
    v = np.zeros((nb * B, H, d))
    for j in range(nb):
        v[j * B:(j + 1) * B, 0, j] = rng.normal(size=B)
    idx = np.tile(np.array([0, 1], dtype=np.int32), (H, nb, 1))
    _, lse = oracle.sparse_attention(q, k, v, idx, B)
    np.testing.assert_allclose(lse, math.log(budget * B), rtol=1e-14)
    drift, jset = oracle.block_drift(q, k, v, idx, lse, B)
    for i in range(nb):
        for r, j in enumerate(range(2, nb)):
            col_sum = v[j * B:(j + 1) * B, 0, j].sum()
            expect = math.sqrt(B) * abs(col_sum) / (budget * B)
            assert drift[0, i, r] == pytest.approx(expect, rel=1e-12)
        assert jset[0, i] == pytest.approx(math.sqrt((drift[0, i] ** 2).sum()), rel=1e-12)


# --------------------------------------------------------------------------
# Layout-aware variant: padding and special tokens
# --------------------------------------------------------------------------

def _layout_case(seed=21, views=3, tpv=16, real=13, n_special=2, B=4, H=2, d=16):
    rng = np.random.default_rng(seed)
    n = views * tpv
    q = rng.normal(size=(n, H, d))
    k = rng.normal(size=(n, H, d))
    v = rng.normal(size=(n, H, d))
    valid, special = oracle.view_layout(n, tpv, real, n_special)
    return q, k, v, valid, special, B


def test_layout_reduces_to_the_plain_path_without_padding_or_special_tokens():
    q, k, v, _, _, B = _layout_case()
    n = q.shape[0]
    valid = np.ones(n, dtype=bool)
    special = np.zeros(n, dtype=bool)
    nb, budget = n // B, 5
    idx = oracle.select_blocks_layout(q, k, B, budget, valid, special)
    assert (idx == oracle.select_blocks(q, k, None, B, budget)).all()
    for h, i in [(0, 0), (1, 5), (0, nb - 1)]:
        o, l = oracle.sparse_attention_layout_block(q, k, v, idx[h, i], h, i, B, valid, special)
        o2, l2 = oracle.sparse_attention_block(q, k, v, idx[h, i], h, i, B)
        assert np.allclose(o, o2, atol=1e-12) and np.allclose(l, l2, atol=1e-12)
        dr, jv = oracle.drift_layout_block(q, k, v, idx[h, i], l, h, i, B, valid, special)
        dr2, jv2 = oracle.drift_block(q, k, v, idx[h, i], l2, h, i, B)
        assert np.allclose(dr, dr2, atol=1e-12) and abs(jv - jv2) < 1e-12


def test_padding_values_change_nothing():
    q, k, v, valid, special, B = _layout_case()
    rng = np.random.default_rng(5)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    pad = ~valid
    for x in (q2, k2, v2):
        x[pad] = rng.normal(size=x[pad].shape) * 100.0
    nb, budget = q.shape[0] // B, 4
    idx = oracle.select_blocks_layout(q, k, B, budget, valid, special)
    assert (idx == oracle.select_blocks_layout(q2, k2, B, budget, valid, special)).all()
    for h in range(q.shape[1]):
        for i in range(nb):
            o, l = oracle.sparse_attention_layout_block(q, k, v, idx[h, i], h, i, B, valid, special)
            o2, l2 = oracle.sparse_attention_layout_block(q2, k2, v2, idx[h, i], h, i, B, valid,
                                                          special)
            assert np.allclose(o, o2, atol=1e-12) and np.array_equal(np.isinf(l), np.isinf(l2))
            dr, jv = oracle.drift_layout_block(q, k, v, idx[h, i], l, h, i, B, valid, special)
            dr2, jv2 = oracle.drift_layout_block(q2, k2, v2, idx[h, i], l2, h, i, B, valid, special)
            assert np.allclose(dr, dr2, atol=1e-10) and abs(jv - jv2) < 1e-10


def test_special_queries_attend_densely_and_padding_queries_write_nothing():
    q, k, v, valid, special, B = _layout_case()
    n, H, d = q.shape
    idx = oracle.select_blocks_layout(q, k, B, 2, valid, special)
    for h in range(H):
        kv = torch.tensor(k[valid, h])[None, None]
        vv = torch.tensor(v[valid, h])[None, None]
        for i in range(n // B):
            o, l = oracle.sparse_attention_layout_block(q, k, v, idx[h, i], h, i, B, valid, special)
            for r in range(B):
                t = i * B + r
                if special[t]:
                    ref = F.scaled_dot_product_attention(torch.tensor(q[t, h])[None, None, None],
                                                         kv, vv)[0, 0, 0].numpy()
                    assert np.allclose(o[r], ref, atol=1e-12)
                    s = torch.tensor(k[valid, h]) @ torch.tensor(q[t, h]) / math.sqrt(d)
                    assert abs(l[r] - float(torch.logsumexp(s, 0))) < 1e-12
                if not valid[t]:
                    assert (o[r] == 0).all() and l[r] == -np.inf


def test_pooling_averages_valid_tokens_only():
    B, H, d = 8, 2, 4
    x = np.full((2 * B, H, d), 1e6)                      # padding: huge values
    x[:5] = 0.375                                        # five valid tokens of block 0
    x[B:B + 8] = np.arange(8, dtype=float)[:, None, None] / 4.0
    valid = np.zeros(2 * B, dtype=bool)
    valid[:5] = True
    valid[B:] = True
    pooled, counts = oracle.pool_blocks_valid(x, B, valid)
    assert list(counts) == [5, 8]
    assert (pooled[:, 0] == 0.375).all()
    assert (pooled[:, 1] == 7.0 / 8.0).all()             # mean of 0, 1/4, ..., 7/4
    empty, c0 = oracle.pool_blocks_valid(x, B, np.zeros(2 * B, dtype=bool))
    assert (empty == 0).all() and (c0 == 0).all()


def test_special_only_key_blocks_are_always_kept():
    # Blocks of 4 tokens; the first block of every 12-token view holds only
    # the 4 special tokens.  Their keys point away from every query, so their
    # logits are the lowest of each row, yet they are kept.
    rng = np.random.default_rng(31)
    views, tpv, B, H, d = 3, 12, 4, 1, 8
    n = views * tpv
    q = np.abs(rng.normal(size=(n, H, d))) + 1.0
    k = np.abs(rng.normal(size=(n, H, d))) + 1.0
    valid, special = oracle.view_layout(n, tpv, tpv, 4)
    k[special] = -5.0
    idx, sc = oracle.select_blocks_layout(q, k, B, 4, valid, special, return_scores=True)
    forced = [j for j in range(n // B) if sc["forced"][j]]
    assert forced == [0, 3, 6]
    for i in range(n // B):
        assert set(forced) <= set(idx[0, i].tolist())
        assert all(sc["logits"][0, i, j] == sc["logits"][0, i].min() or j not in forced
                   for j in forced)
        others = [j for j in idx[0, i].tolist() if j not in forced]
        rest = [j for j in np.argsort(-sc["logits"][0, i], kind="stable") if j not in forced]
        assert others == sorted(rest[:1])


def test_empty_key_blocks_are_never_preferred_to_non_empty_ones():
    # Views of 12 tokens with 8 real ones and blocks of 4: block 2 of every
    # view (positions 8..11) holds only padding and pools to the zero vector,
    # so its logit is exactly 0.  Every valid key points away from every
    # query, so every non-empty block has a negative logit: ranked like the
    # others, the empty blocks would be the top of each row.  The expected
    # kept set comes from plain means over the valid tokens and a stable
    # sort of the non-empty blocks alone.
    rng = np.random.default_rng(17)
    views, tpv, real, B, H, d = 3, 12, 8, 4, 2, 8
    n = views * tpv
    q = np.abs(rng.normal(size=(n, H, d))) + 0.5
    k = -(np.abs(rng.normal(size=(n, H, d))) + 0.5)
    valid, special = oracle.view_layout(n, tpv, real, 0)
    nb, budget = n // B, 4
    empty = [j for j in range(nb) if not valid[j * B:(j + 1) * B].any()]
    assert empty == [2, 5, 8]
    idx = oracle.select_blocks_layout(q, k, B, budget, valid, special)
    for h in range(H):
        kbar = {j: k[j * B:(j + 1) * B][valid[j * B:(j + 1) * B], h].mean(axis=0)
                for j in range(nb) if j not in empty}
        for i in range(nb):
            toks = valid[i * B:(i + 1) * B]
            if not toks.any():
                continue
            qbar = q[i * B:(i + 1) * B][toks, h].mean(axis=0)
            cand = sorted(kbar)
            s = np.array([qbar @ kbar[j] for j in cand]) / math.sqrt(d)
            assert (s < 0).all()
            order = np.argsort(-s, kind="stable")[:budget]
            assert idx[h, i].tolist() == sorted(cand[o] for o in order)
            assert not set(empty) & set(idx[h, i].tolist())


def test_layout_drift_reconstructs_dense_attention_over_valid_keys():
    q, k, v, valid, special, B = _layout_case(seed=41)
    n, H, d = q.shape
    idx = oracle.select_blocks_layout(q, k, B, 4, valid, special)
    for h in range(H):
        for i in range(n // B):
            o, l = oracle.sparse_attention_layout_block(q, k, v, idx[h, i], h, i, B, valid, special)
            kept_tok = np.zeros(n, dtype=bool)
            for j in idx[h, i]:
                kept_tok[j * B:(j + 1) * B] = True
            drop_tok = valid & ~kept_tok
            for r in range(B):
                t = i * B + r
                if not valid[t] or special[t]:
                    continue
                # dense over the valid keys, from torch only
                dense = F.scaled_dot_product_attention(
                    torch.tensor(q[t, h])[None, None, None], torch.tensor(k[valid, h])[None, None],
                    torch.tensor(v[valid, h])[None, None])[0, 0, 0].numpy()
                s = (k[drop_tok, h] @ q[t, h]) / math.sqrt(d)
                w = np.exp(s - l[r])
                c_sum = w @ v[drop_tok, h]
                assert np.allclose((o[r] + c_sum) / (1.0 + w.sum()), dense, atol=1e-10)
            # every C_j row of a special or padding query is zero: a block of
            # only such queries has zero drift
            dr, jv = oracle.drift_layout_block(q, k, v, idx[h, i], l, h, i, B, valid, special)
            rows = np.arange(i * B, (i + 1) * B)
            if not (valid[rows] & ~special[rows]).any():
                assert (dr == 0).all() and jv == 0.0
            else:
                assert jv <= dr.sum() + 1e-12
    # a block made only of special queries: zero drift, whatever it drops
    vq, sq = oracle.view_layout(n, 16, 16, 8)
    idx2 = oracle.select_blocks_layout(q, k, B, 2, vq, sq)
    o, l = oracle.sparse_attention_layout_block(q, k, v, idx2[0, 0], 0, 0, B, vq, sq)
    dr, jv = oracle.drift_layout_block(q, k, v, idx2[0, 0], l, 0, 0, B, vq, sq)
    assert dr.shape[0] > 0 and (dr == 0).all() and jv == 0.0


# --------------------------------------------------------------------------
# ReSS drift-based selection with restoration (pooled contributions)
# --------------------------------------------------------------------------

def test_pooled_contribution_is_probability_times_pooled_value():
    w, q, k, v = _tiny_inputs()
    c = oracle.pooled_contributions(q, k, v, w.block)
    B = w.block
    tq, tk, tv = (torch.tensor(x) for x in (q, k, v))
    nb = tq.shape[0] // B
    qb = tq.view(nb, B, *tq.shape[1:]).mean(1)      # [nb, H, d]
    kb = tk.view(nb, B, *tk.shape[1:]).mean(1)
    vb = tv.view(nb, B, *tv.shape[1:]).mean(1)
    for h in range(tq.shape[1]):
        p = torch.softmax(qb[:, h] @ kb[:, h].T / 8.0, dim=-1)      # [nb, nb]
        ref = p[:, :, None] * vb[None, :, h]
        assert np.allclose(c[h], ref.numpy(), atol=1e-14)


def test_restoration_closed_form_two_rounds():
    # Four blocks in d = 2, budget 2.  Drift scores 3, 2.9, 1, 1 keep {0, 1},
    # so D = {2, 3} and J = 2.  Round 1: the best swap restores block 2 and
    # drops block 1 (J = 1.9; restoring 3 instead ties and loses on index).
    # Round 2: restore 3, drop 0: D = {0, 1}, J = |3 - 2.9| = 0.1, which no
    # further swap improves; it is also the best of all six drop sets.
    c = np.array([[3.0, 0.0], [-2.9, 0.0], [1.0, 0.0], [1.0, 0.0]])
    kept, j0, j = oracle.restore_row(c, 2, rounds=1)
    assert kept.tolist() == [0, 2] and j0 == 2.0 and abs(j - 1.9) < 1e-12
    kept, j0, j = oracle.restore_row(c, 2, rounds=4)
    assert kept.tolist() == [2, 3] and abs(j - 0.1) < 1e-12
    best = min(abs(c[list(set(range(4)) - set(s))].sum(0)[0])
               for s in itertools.combinations(range(4), 2))
    assert abs(best - 0.1) < 1e-12
    kept0, _, j00 = oracle.restore_row(c, 2, rounds=0)
    assert kept0.tolist() == [0, 1] and j00 == 2.0


def test_restoration_without_rounds_is_top_drift_score():
    w, q, k, v = _tiny_inputs()
    idx, j0, j1 = oracle.select_blocks_restore(q, k, v, w.block, w.budget, rounds=0)
    c = oracle.pooled_contributions(q, k, v, w.block)
    score = torch.linalg.vector_norm(torch.tensor(c), dim=-1).numpy()
    ref = np.sort(np.argsort(-score, axis=-1, kind="stable")[..., :w.budget], axis=-1)
    assert (idx == ref).all() and np.array_equal(j0, j1)


def test_one_round_takes_the_best_single_swap_brute_force():
    # nb = 8, budget 4, cand = 8 covers every pair: one round must land on the
    # best drop set one swap away from the initial set (when it beats J0).
    w, q, k, v = _tiny_inputs()
    c = oracle.pooled_contributions(q, k, v, w.block)
    nb = c.shape[1]
    for h in range(c.shape[0]):
        for i in range(nb):
            row = torch.tensor(c[h, i])
            score = torch.linalg.vector_norm(row, dim=-1).numpy()
            k0 = set(np.argsort(-score, kind="stable")[:w.budget].tolist())

            def jd(kept):
                drop = [j for j in range(nb) if j not in kept]
                return float(torch.linalg.vector_norm(row[drop].sum(0)))
            cands = [(jd((k0 - {a}) | {b}), b, a) for b in range(nb) if b not in k0 for a in k0]
            jbest, b, a = min(cands)
            kept, j0, j1 = oracle.restore_row(c[h, i], w.budget, rounds=1)
            assert abs(j0 - jd(k0)) < 1e-13
            if jbest < j0:
                assert kept.tolist() == sorted((k0 - {a}) | {b}) and abs(j1 - jbest) < 1e-13
            else:
                assert kept.tolist() == sorted(k0) and j1 == j0


def test_restoration_never_raises_j_and_never_beats_the_optimum():
    w, q, k, v = _tiny_inputs()
    c = oracle.pooled_contributions(q, k, v, w.block)
    nb = c.shape[1]
    idx, j0, j1 = oracle.select_blocks_restore(q, k, v, w.block, w.budget, rounds=4)
    assert (j1 <= j0).all()
    for h in range(c.shape[0]):
        for i in range(nb):
            row = torch.tensor(c[h, i])
            opt = min(float(torch.linalg.vector_norm(row[list(set(range(nb)) - set(s))].sum(0)))
                      for s in itertools.combinations(range(nb), w.budget))
            assert j1[h, i] >= opt - 1e-13
            drop = [j for j in range(nb) if j not in idx[h, i]]
            assert abs(j1[h, i] - float(torch.linalg.vector_norm(row[drop].sum(0)))) < 1e-13
            assert len(set(idx[h, i].tolist())) == w.budget and (np.diff(idx[h, i]) > 0).all()


def test_restoration_stops_at_a_local_minimum():
    # d = 1, budget 2: drift scores 1, 0, 4, 3, 0 keep {2, 3}; D = {0, 1, 4}
    # sums to -1 (J = 1).  Every single swap gives |sum| >= 3, so restoration
    # stops there, although the drop set {0, 2, 3} sums to 0.
    c = np.array([[-1.0], [0.0], [4.0], [-3.0], [0.0]])
    for s in itertools.combinations(range(5), 2):
        if set(s) == {2, 3}:
            continue
        if len(set(s) & {2, 3}) == 1:          # one swap away
            assert abs(c[list(set(range(5)) - set(s))].sum()) >= 3.0
    kept, j0, j = oracle.restore_row(c, 2, rounds=4)
    assert kept.tolist() == [2, 3] and j0 == 1.0 and j == 1.0
    assert abs(c[[0, 2, 3]].sum()) == 0.0


def test_restoration_candidates_are_the_largest_gains_and_smallest_costs():
    # d = 1, budget 2, one candidate per side.  Scores 5, 5, 4, 3, 4, 0 keep
    # {0, 1}; D = {2, 3, 4, 5} sums to T = 11.  Gains 2 T c_b - c_b^2 are 72,
    # 57, 72, 0: block 2 (72, lower index than 4).  Costs 2 T c_a + c_a^2 are
    # -85, -85: block 0.  The swap gives 11 - 4 - 5 = 2 < 11.
    c = np.array([[-5.0], [-5.0], [4.0], [3.0], [4.0], [0.0]])
    kept, j0, j = oracle.restore_row(c, 2, rounds=1, cand=1)
    assert kept.tolist() == [1, 2] and j0 == 11.0 and j == 2.0


# --------------------------------------------------------------------------
# VASC: pair contrast, demand, memory
# --------------------------------------------------------------------------

def test_block_pairs_and_pair_contrast_closed_form():
    # nb = 5, d = 4: pairs (0, 1), (2, 3) and the singleton 4.  Pooled values
    # 0 and 2 (every dimension) differ by 2 in each of the 4 dimensions: RMS 2
    # (the L2 norm would be 4).  Blocks 2 and 3 differ by 2 in one dimension:
    # RMS sqrt(4 / 4) = 1.  The singleton has contrast 0.
    pair_of, size = oracle.block_pairs(5)
    assert pair_of.tolist() == [0, 0, 1, 1, 2] and size.tolist() == [2, 2, 1]
    vbar = np.array([[[0.0, 0, 0, 0], [2, 2, 2, 2], [1, 0, 0, 0], [1, 0, 0, 2], [9, 9, 9, 9]]])
    assert np.array_equal(oracle.pair_contrast(vbar), np.array([[2.0, 1.0, 0.0]]))
    pair_of, size = oracle.block_pairs(4)
    assert pair_of.tolist() == [0, 0, 1, 1] and size.tolist() == [2, 2]


def test_pair_contrast_matches_torch_on_pooled_tokens():
    rng = np.random.default_rng(31)
    B, nb, H, d = 8, 7, 3, 16
    v = rng.normal(size=(nb * B, H, d))
    vb = torch.from_numpy(v).view(nb, B, H, d).mean(dim=1)          # [nb, H, d]
    ref = (vb[0:nb - 1:2] - vb[1:nb:2]).pow(2).mean(dim=-1).sqrt()  # [3, H]
    got = oracle.pair_contrast(oracle.pool_blocks(v, B))
    np.testing.assert_allclose(got[:, :3], ref.T.numpy(), rtol=1e-13, atol=1e-15)
    assert (got[:, 3] == 0.0).all()


def test_demand_closed_forms():
    # One row, nb = 4, p = (1/2, 1/4, 1/8, 1/8).
    p = np.array([[[0.5, 0.25, 0.125, 0.125]]])
    ones = np.ones((1, 2))
    # Contrast one: capacity 2 gives 2 p = (1, 1/2, 1/4, 1/4), nothing clipped.
    np.testing.assert_allclose(oracle.vasc_demand(p, ones, [2]), [[[1.0, 0.5, 0.25, 0.25]]],
                               rtol=0, atol=1e-15)
    np.testing.assert_allclose(oracle.vasc_demand(p, 5 * ones, [2], value_aware=False),
                               [[[1.0, 0.5, 0.25, 0.25]]], rtol=0, atol=1e-15)
    # Capacity 3: 3 p = (3/2, 3/4, 3/8, 3/8); the first entry clips to one.
    np.testing.assert_allclose(oracle.vasc_demand(p, ones, [3]), [[[1.0, 0.75, 0.375, 0.375]]],
                               rtol=0, atol=1e-15)
    # Contrast (1, 2) multiplies: d = (1/2, 1/4, 1/4, 1/4), total 5/4, so
    # capacity 2 gives (4/5, 2/5, 2/5, 2/5).
    rho = np.array([[1.0, 2.0]])
    np.testing.assert_allclose(oracle.vasc_demand(p, rho, [2]), [[[0.8, 0.4, 0.4, 0.4]]],
                               rtol=0, atol=1e-15)
    # A pair without contrast has no demand.
    np.testing.assert_allclose(oracle.vasc_demand(p, np.array([[0.0, 1.0]]), [1]),
                               [[[0.0, 0.0, 0.5, 0.5]]], rtol=0, atol=1e-15)


def test_demand_invariants_on_tiny():
    w, q, k, v = _tiny_inputs()
    probs = oracle.selection_scores(q, k, None, w.block, 0.0)["probs"]
    rho = oracle.pair_contrast(oracle.pool_blocks(v, w.block))
    budgets = [3, 5][:probs.shape[0]]
    a = oracle.vasc_demand(probs, rho, budgets)
    assert (a >= 0).all() and (a <= 1.0).all()
    for h, c in enumerate(budgets):
        tot = a[h].sum(axis=-1)
        assert (tot <= c + 1e-12).all()
        d = probs[h] * rho[h][np.arange(probs.shape[-1]) // 2][None, :]
        unclipped = (c * d / d.sum(-1, keepdims=True)).max(-1) <= 1.0
        np.testing.assert_allclose(tot[unclipped], c, rtol=1e-13)


def test_memory_ranking_copy_normalises_each_head_by_its_largest_balance():
    mem = np.array([[0.0, 2.0, 1.0], [0.0, 0.0, 0.0], [3.0, 0.0, 6.0]])
    np.testing.assert_array_equal(oracle.memory_ranking_copy(mem),
                                  [[0.0, 1.0, 0.5], [0.0, 0.0, 0.0], [0.5, 0.0, 1.0]])


def test_pair_means_average_over_query_blocks_and_children():
    # H = 1, two query blocks, nb = 3: pair 0 = blocks 0 and 1, block 2 alone.
    x = np.array([[[1.0, 2.0, 3.0], [3.0, 4.0, 5.0]]])
    np.testing.assert_array_equal(oracle.pair_means(x), [[2.5, 4.0]])


def _vasc_hand_inputs():
    # B = 4, nb = 4, H = 1, d = 4.  Q = 0: every pooled logit is 0 and every
    # probability 1/4.  Pooled values 0, 2, 0, 1: pair contrasts 2 and 1.
    B, nb, d = 4, 4, 4
    q = np.zeros((B * nb, 1, d))
    k = np.random.default_rng(5).normal(size=(B * nb, 1, d))
    v = np.zeros((B * nb, 1, d))
    v[B:2 * B] = 2.0
    v[3 * B:] = 1.0
    return q, k, v, B


def test_vasc_hand_worked_layers():
    # Capacity 1.  Demand d = (1/4)(2, 2, 1, 1), total 3/2: a = (1/3, 1/3, 1/6,
    # 1/6) in every row.  Pair means: D = (1/3, 1/6).
    #  layer 1, no memory: block 0 (tie with 1, lower index); S = (1/2, 0);
    #           memory max(0, (1/3 - 1/2, 1/6)) = (0, 1/6).
    #  layer 2: ranking copy (0, 1), scores (1/3, 1/3, 7/6, 7/6): block 2;
    #           S = (0, 1/2); memory (0 + 1/3, 1/6 + 1/6 - 1/2 -> 0) = (1/3, 0).
    #  layer 3: copy (1, 0): block 0; memory (1/3 + 1/3 - 1/2, 0 + 1/6) = (1/6, 1/6).
    #  layer 4: copy (1, 1): scores (4/3, 4/3, 7/6, 7/6): block 0;
    #           memory (1/6 + 1/3 - 1/2, 1/6 + 1/6) = (0, 1/3).
    q, k, v, B = _vasc_hand_inputs()
    expect = [(0, [0.0, 1 / 6]), (2, [1 / 3, 0.0]), (0, [1 / 6, 1 / 6]), (0, [0.0, 1 / 3])]
    mem = None
    for layer, (block, mem_ref) in enumerate(expect):
        idx, mem, info = oracle.select_blocks_vasc(q, k, v, B, [1], 2, mem)
        np.testing.assert_allclose(info["demand"][0], np.tile([1 / 3, 1 / 3, 1 / 6, 1 / 6], (4, 1)),
                                   rtol=0, atol=1e-15)
        np.testing.assert_allclose(info["D"], [[1 / 3, 1 / 6]], rtol=0, atol=1e-15)
        assert (idx[0] == block).all(), (layer, idx[0])       # kept block, repeated to capacity
        np.testing.assert_allclose(mem, [mem_ref], rtol=0, atol=1e-15)


def test_vasc_without_memory_or_contrast_is_the_pooled_topk():
    w, q, k, v = _tiny_inputs()
    H = q.shape[1]
    budgets = [w.budget] * H
    idx, _, _ = oracle.select_blocks_vasc(q, k, v, w.block, budgets, w.budget, None,
                                          value_aware=False)
    assert np.array_equal(idx, oracle.select_blocks(q, k, None, w.block, w.budget, 0.0))


def test_vasc_without_memory_keeps_the_top_modulated_relevance():
    # The clip changes no set: at most c_h entries of a row reach one, and they
    # are the c_h largest p * rho.  Reference from torch, ranked by brute force.
    w, q, k, v = _tiny_inputs()
    B, H = w.block, q.shape[1]
    budgets = [3, 5][:H]
    idx, _, _ = oracle.select_blocks_vasc(q, k, v, B, budgets, max(budgets), None)
    tq, tk, tv = (torch.tensor(x) for x in (q, k, v))
    nb = tq.shape[0] // B
    qb, kb, vb = (t.view(nb, B, *t.shape[1:]).mean(1) for t in (tq, tk, tv))
    for h in range(H):
        p = torch.softmax(qb[:, h] @ kb[:, h].T / 8.0, dim=-1)
        rho = (vb[0::2, h] - vb[1::2, h]).pow(2).mean(-1).sqrt()
        d = (p * rho.repeat_interleave(2)[None, :nb]).numpy()
        for i in range(nb):
            ref = _brute_force_topk(d[i], budgets[h])
            assert idx[h, i, :budgets[h]].tolist() == list(ref)
            assert (idx[h, i, budgets[h]:] == ref[-1]).all()


def test_vasc_with_memory_equals_brute_force_and_conserves_service():
    w, q, k, v = _tiny_inputs()
    H, B = q.shape[1], w.block
    nb = q.shape[0] // B
    budgets = [2, 4][:H]
    mem_in = np.random.default_rng(8).uniform(0.0, 0.3, size=(H, (nb + 1) // 2))
    idx, mem, info = oracle.select_blocks_vasc(q, k, v, B, budgets, 4, mem_in)
    for h in range(H):
        for i in range(nb):
            ref = _brute_force_topk(info["score"][h, i], budgets[h])
            assert idx[h, i, :budgets[h]].tolist() == list(ref)
    _, size = oracle.block_pairs(nb)
    for h, c in enumerate(budgets):
        # Every row executes exactly c_h children: sum_p size_p S_p = c_h.
        assert abs((info["S"][h] * size).sum() - c) < 1e-12
        assert (info["D"][h] * size).sum() <= c + 1e-12
    assert (mem >= 0).all()
    np.testing.assert_allclose(mem, np.maximum(0.0, mem_in + info["D"] - info["S"]), rtol=0,
                               atol=0)
