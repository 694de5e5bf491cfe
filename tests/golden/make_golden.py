"""Write the oracle regression fixture ``oracle_tiny.json``.

The pages print no worked example for this path, so the fixture is not a pin:
it records what the oracle returns on the seeded tiny workload, so that any
later change to the oracle's arithmetic shows up as a diff that its commit has
to justify.  Only ``oracle/`` and the seeded input generator are called.

    python tests/golden/make_golden.py
"""

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
from block_sparse_global_mean_b200 import workloads  # noqa: E402


def main():
    w = workloads.WORKLOADS["tiny"]
    q, k, v = (t.to(torch.float64).numpy() for t in workloads.generate(w))
    idx, sc = oracle.select_blocks(q, k, v, w.block, w.budget, 0.0, return_scores=True)
    out, lse = oracle.sparse_attention(q, k, v, idx, w.block)
    drift, jset = oracle.block_drift(q, k, v, idx, lse, w.block)
    rows = [0, 63, 64, 300, 511]
    fixture = {
        "workload": "tiny",
        "source": "oracle/ress_oracle.py on workloads.generate(WORKLOADS['tiny'])",
        "idx": idx.tolist(),
        "logits_row_h0_i0": sc["logits"][0, 0].tolist(),
        "out_rows": rows,
        "out_h1": out[rows, 1, :].tolist(),
        "lse_h0": lse[0, rows].tolist(),
        "drift_h0_i0": drift[0, 0].tolist(),
        "J": jset.tolist(),
    }
    # CDF threshold on the same pooled probabilities.
    for tau in (0.5, 0.9):
        counts, cidx = oracle.select_blocks_cdf(q, k, w.block, tau, w.n_blocks)
        fixture[f"cdf_counts_tau{tau}"] = counts.tolist()
        fixture[f"cdf_idx_tau{tau}"] = cidx.tolist()
    # Layout-aware variant: 2 views of 256 tokens, the last 20 of each padding,
    # the first 5 special.
    valid, special = oracle.view_layout(w.n_tokens, 256, 236, 5)
    lidx = oracle.select_blocks_layout(q, k, w.block, w.budget, valid, special)
    fixture["layout_idx"] = lidx.tolist()
    lo, ll = oracle.sparse_attention_layout_block(q, k, v, lidx[1, 3], 1, 3, w.block, valid, special)
    fixture["layout_out_h1_i3_rows"] = [0, 4, 5, 63]
    fixture["layout_out_h1_i3"] = lo[[0, 4, 5, 63]].tolist()
    fixture["layout_lse_h1_i3"] = [float(x) for x in ll]
    ld, lj = oracle.drift_layout_block(q, k, v, lidx[1, 3], ll, 1, 3, w.block, valid, special)
    fixture["layout_drift_h1_i3"] = ld.tolist()
    fixture["layout_J_h1_i3"] = lj
    # Restoration-based selection (4 rounds, 8 candidates).
    ridx, rj0, rj1 = oracle.select_blocks_restore(q, k, v, w.block, w.budget, 4, 8)
    fixture["restore_idx"] = ridx.tolist()
    fixture["restore_j_init"] = rj0.tolist()
    fixture["restore_j_final"] = rj1.tolist()
    # VASC: three layers (layer l drawn with seed + 1000 (l + 1)), budgets 3 and
    # 5, rows of 6, the memory carried from layer to layer.
    mem = None
    for layer in range(3):
        ql, kl, vl = (t.to(torch.float64).numpy()
                      for t in workloads.generate(w, seed=w.seed + 1000 * (layer + 1)))
        vidx, mem, _ = oracle.select_blocks_vasc(ql, kl, vl, w.block, [3, 5], 6, mem)
        fixture[f"vasc_idx_layer{layer}"] = vidx.tolist()
        fixture[f"vasc_memory_layer{layer}"] = mem.tolist()
    with open(os.path.join(HERE, "oracle_tiny.json"), "w") as f:
        json.dump(fixture, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
