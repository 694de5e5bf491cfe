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
