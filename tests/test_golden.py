"""The oracle still reproduces its recorded output on the tiny workload."""

import json
import os

import numpy as np
import torch

import oracle
from block_sparse_global_mean_b200 import workloads

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_reproduces_recorded_tiny_outputs():
    with open(os.path.join(HERE, "oracle_tiny.json")) as f:
        g = json.load(f)
    w = workloads.WORKLOADS["tiny"]
    q, k, v = (t.to(torch.float64).numpy() for t in workloads.generate(w))
    idx, sc = oracle.select_blocks(q, k, v, w.block, w.budget, 0.0, return_scores=True)
    np.testing.assert_array_equal(idx, np.array(g["idx"]))
    np.testing.assert_allclose(sc["logits"][0, 0], g["logits_row_h0_i0"], rtol=1e-12)
    out, lse = oracle.sparse_attention(q, k, v, idx, w.block)
    rows = g["out_rows"]
    np.testing.assert_allclose(out[rows, 1, :], g["out_h1"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse[0, rows], g["lse_h0"], rtol=1e-12)
    drift, jset = oracle.block_drift(q, k, v, idx, lse, w.block)
    np.testing.assert_allclose(drift[0, 0], g["drift_h0_i0"], rtol=1e-12)
    np.testing.assert_allclose(jset, g["J"], rtol=1e-12)


def test_oracle_reproduces_recorded_cdf_and_layout_outputs():
    with open(os.path.join(HERE, "oracle_tiny.json")) as f:
        g = json.load(f)
    w = workloads.WORKLOADS["tiny"]
    q, k, v = (t.to(torch.float64).numpy() for t in workloads.generate(w))
    for tau in (0.5, 0.9):
        counts, cidx = oracle.select_blocks_cdf(q, k, w.block, tau, w.n_blocks)
        np.testing.assert_array_equal(counts, np.array(g[f"cdf_counts_tau{tau}"]))
        np.testing.assert_array_equal(cidx, np.array(g[f"cdf_idx_tau{tau}"]))
    valid, special = oracle.view_layout(w.n_tokens, 256, 236, 5)
    lidx = oracle.select_blocks_layout(q, k, w.block, w.budget, valid, special)
    np.testing.assert_array_equal(lidx, np.array(g["layout_idx"]))
    lo, ll = oracle.sparse_attention_layout_block(q, k, v, lidx[1, 3], 1, 3, w.block, valid,
                                                  special)
    np.testing.assert_allclose(lo[g["layout_out_h1_i3_rows"]], g["layout_out_h1_i3"],
                               rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(ll, g["layout_lse_h1_i3"], rtol=1e-12)
    ld, lj = oracle.drift_layout_block(q, k, v, lidx[1, 3], ll, 1, 3, w.block, valid, special)
    np.testing.assert_allclose(ld, g["layout_drift_h1_i3"], rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(lj, g["layout_J_h1_i3"], rtol=1e-12)


def test_oracle_reproduces_recorded_restore_and_vasc_outputs():
    with open(os.path.join(HERE, "oracle_tiny.json")) as f:
        g = json.load(f)
    w = workloads.WORKLOADS["tiny"]
    q, k, v = (t.to(torch.float64).numpy() for t in workloads.generate(w))
    ridx, rj0, rj1 = oracle.select_blocks_restore(q, k, v, w.block, w.budget, 4, 8)
    np.testing.assert_array_equal(ridx, np.array(g["restore_idx"]))
    np.testing.assert_allclose(rj0, g["restore_j_init"], rtol=1e-12)
    np.testing.assert_allclose(rj1, g["restore_j_final"], rtol=1e-12)
    mem = None
    for layer in range(3):
        ql, kl, vl = (t.to(torch.float64).numpy()
                      for t in workloads.generate(w, seed=w.seed + 1000 * (layer + 1)))
        vidx, mem, _ = oracle.select_blocks_vasc(ql, kl, vl, w.block, [3, 5], 6, mem)
        np.testing.assert_array_equal(vidx, np.array(g[f"vasc_idx_layer{layer}"]))
        np.testing.assert_allclose(mem, g[f"vasc_memory_layer{layer}"], rtol=1e-12, atol=1e-15)
