"""VASC selection (value-aware demand, per-head budgets, cross-layer memory)
on the GPU against the oracle, layer after layer.

Each layer's oracle call takes the memory the GPU carried in (float32, as the
GPU stores it), so that a near-tie decided differently in one layer cannot
leak into the next.  The kept sets must equal the oracle's except for rows
whose differing blocks score within MARGIN of the row's c_h-th score; the
demand means D must match the oracle's; the service means S and the settled
memory must match what the GPU's own mask implies (exact counts).  Outputs
start poisoned."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_global_mean_b200 import workloads
from tests.parity import np64, poison, sample_rows

pytestmark = pytest.mark.gpu

MARGIN = 1e-5          # ranking-score units (demand <= 1 plus memory copy <= 1)
MAX_EXCUSED = 0.05     # fraction of rows allowed to differ within the margin
D_ABS = 2e-6           # demand means: float32 demand, fixed-point sums
S_ABS = 1e-7           # service means: exact counts, stored as float32
MEM_ABS = 4e-6


def _layer_inputs(w, layer, device="cuda", n_tokens=None):
    q, k, v = workloads.generate(w, device=device, seed=w.seed + 1000 * (layer + 1))
    if n_tokens is not None:
        q, k, v = (t[:n_tokens].contiguous() for t in (q, k, v))
    return q, k, v


def _run(ress, q, k, v, budgets, block, capacity, mem, value_aware=True, reset=False):
    h, nb = q.shape[1], q.shape[0] // block
    pairs = ress.vasc_pairs(nb)
    idx = poison((h, nb, capacity), torch.int32, q.device)
    dem = poison((h, pairs), torch.float32, q.device)
    ser = poison((h, pairs), torch.float32, q.device)
    ress.ress_select_blocks_vasc(q, k, v if value_aware else None, budgets, block, capacity,
                                 memory=mem, value_aware=value_aware, reset=reset, idx=idx,
                                 demand=dem, service=ser)
    status, detail = ress.ress_check_device_errors()
    assert status == 0, (status, detail)
    return idx.cpu().numpy(), dem.cpu().numpy().astype(np.float64), ser.cpu().numpy().astype(
        np.float64)


def _check_layer(q, k, v, block, budgets, capacity, mem_in, idx, dem, ser, mem_out,
                 value_aware=True, rows=None):
    """Compares one GPU layer with the oracle fed the same memory.  Returns the
    number of rows whose kept set differs (within the margin)."""
    q64, k64, v64 = np64(q), np64(k), np64(v) if v is not None else None
    ref_idx, _, info = oracle.select_blocks_vasc(q64, k64, v64, block, budgets, capacity, mem_in,
                                                 value_aware=value_aware)
    h_count, nb, _ = ref_idx.shape
    mask = np.zeros((h_count, nb, nb))
    differ = 0
    for h in range(h_count):
        c = budgets[h]
        for i in range(nb):
            kept = idx[h, i, :c]
            assert np.all(np.diff(kept) > 0) and kept[0] >= 0 and kept[-1] < nb, (h, i, kept)
            assert (idx[h, i, c:] == kept[-1]).all(), (h, i, idx[h, i])
            mask[h, i, kept] = 1.0
            if rows is not None and (h, i) not in rows:
                continue
            a, b = set(kept.tolist()), set(ref_idx[h, i, :c].tolist())
            if a == b:
                continue
            differ += 1
            row = info["score"][h, i]
            kth = np.sort(row)[::-1][c - 1]
            for j in a ^ b:
                assert abs(row[j] - kth) <= MARGIN, (h, i, j, row[j], kth)
    total = h_count * nb if rows is None else len(rows)
    assert differ <= MAX_EXCUSED * total, f"{differ} of {total} rows differ"
    np.testing.assert_allclose(dem, info["D"], rtol=0, atol=D_ABS)
    s_own = oracle.pair_means(mask)
    np.testing.assert_allclose(ser, s_own, rtol=0, atol=S_ABS)
    mem_ref = np.maximum(0.0, mem_in + info["D"] - s_own)
    np.testing.assert_allclose(mem_out, mem_ref, rtol=0, atol=MEM_ABS)
    return differ


def _layers(ress, w, budgets, capacity, layers, value_aware=True, n_tokens=None, block=None):
    block = block or w.block
    mem = None
    for layer in range(layers):
        q, k, v = _layer_inputs(w, layer, n_tokens=n_tokens)
        h, nb = q.shape[1], q.shape[0] // block
        if mem is None:
            mem = poison((h, ress.vasc_pairs(nb)), torch.float32, q.device)   # reset ignores it
            mem_in = np.zeros((h, ress.vasc_pairs(nb)))
            reset = True
        else:
            mem_in = mem.cpu().numpy().astype(np.float64)
            reset = False
        idx, dem, ser = _run(ress, q, k, v, budgets, block, capacity, mem, value_aware, reset)
        mem_out = mem.cpu().numpy().astype(np.float64)
        assert np.isfinite(mem_out).all() and (mem_out >= 0).all()
        _check_layer(q, k, v if value_aware else None, block, budgets, capacity, mem_in, idx, dem,
                     ser, mem_out, value_aware)
    return mem


def test_vasc_tiny_four_layers_per_head_budgets(ress_gpu):
    # float32 inputs, H = 2, nb = 8: budgets 3 and 5, rows padded to 6.
    _layers(ress_gpu, workloads.WORKLOADS["tiny"], [3, 5], 6, layers=4)


def test_vasc_vggt8_three_layers_per_head_budgets(ress_gpu):
    w = workloads.WORKLOADS["vggt8"]
    budgets = [88 - 4 * h for h in range(w.heads)]       # 88 .. 28
    budgets[3] = 1                                       # the smallest budget
    _layers(ress_gpu, w, budgets, 88, layers=3)


def test_vasc_odd_block_count_has_a_singleton(ress_gpu):
    # 175 key blocks: pairs (0, 1) .. (172, 173) and the singleton 174.
    w = workloads.WORKLOADS["vggt8"]
    mem = _layers(ress_gpu, w, [40] * w.heads, 40, layers=2, n_tokens=175 * 64)
    assert mem.shape[1] == 88


def test_vasc_block_128_and_budget_equal_to_capacity(ress_gpu):
    w = workloads.WORKLOADS["vggt8"]
    budgets = [44] * w.heads
    budgets[0] = 1
    _layers(ress_gpu, w, budgets, 44, layers=2, block=128)


def test_vasc_without_contrast_or_memory_is_the_pooled_topk(ress_gpu):
    # Contrast one and no memory: the demand ranks like the pooled
    # probabilities, so the kept sets are those of ress_select_blocks.
    w = workloads.WORKLOADS["vggt8"]
    q, k, v = _layer_inputs(w, 0)
    idx, _, _ = _run(ress_gpu, q, k, v, [w.budget] * w.heads, w.block, w.budget,
                     torch.zeros((w.heads, ress_gpu.vasc_pairs(w.n_blocks)), device="cuda"),
                     value_aware=False, reset=True)
    ref = ress_gpu.ress_select_blocks(q, k, None, w.budget, 0.0, w.block).cpu().numpy()
    same = (idx == ref).all(axis=-1).mean()
    assert same >= 0.99, same
    _layers(ress_gpu, w, [w.budget] * w.heads, w.budget, layers=2, value_aware=False)


def test_vasc_is_deterministic(ress_gpu):
    w = workloads.WORKLOADS["vggt8"]
    q, k, v = _layer_inputs(w, 0)
    pairs = ress_gpu.vasc_pairs(w.n_blocks)
    start = torch.rand((w.heads, pairs), device="cuda") * 0.2
    outs = []
    for _ in range(3):
        mem = start.clone()
        idx, dem, ser = _run(ress_gpu, q, k, v, [60] * w.heads, w.block, 60, mem)
        outs.append((idx, dem, ser, mem.cpu().numpy()))
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert np.array_equal(a, b)


def test_vasc_4096_blocks(ress_gpu):
    # The largest supported block count (N = 262,144, H = 2).
    g = torch.Generator().manual_seed(77)
    n, h = 4096 * 64, 2
    q, k, v = (torch.randn(n, h, 64, generator=g).to("cuda", torch.bfloat16) for _ in range(3))
    mem = torch.rand((h, 2048), generator=g).mul_(0.1).to("cuda")
    mem_in = mem.cpu().numpy().astype(np.float64)
    idx, dem, ser = _run(ress_gpu, q, k, v, [1, 300], 64, 300, mem)
    _check_layer(q, k, v, 64, [1, 300], 300, mem_in, idx, dem, ser,
                 mem.cpu().numpy().astype(np.float64))


def test_vasc_views100_sampled_rows(ress_gpu, wcache):
    # The 100-view workload with a carried memory: the whole mask is checked
    # for validity and its D, S and memory; the kept sets on sampled rows.
    w = workloads.WORKLOADS["views100"]
    q, k, v = wcache.get(w)
    pairs = ress_gpu.vasc_pairs(w.n_blocks)
    mem = (torch.rand((w.heads, pairs), generator=torch.Generator().manual_seed(5)) * 0.05).to("cuda")
    mem_in = mem.cpu().numpy().astype(np.float64)
    budgets = [w.budget - 8 * (h % 4) for h in range(w.heads)]
    idx, dem, ser = _run(ress_gpu, q, k, v, budgets, w.block, w.budget, mem)
    rows = set(sample_rows(w.heads, w.n_blocks, count=96))
    _check_layer(q, k, v, w.block, budgets, w.budget, mem_in, idx, dem, ser,
                 mem.cpu().numpy().astype(np.float64), rows=rows)


def test_vasc_64_heads_with_budgets_from_one_to_capacity(ress_gpu):
    # The head maximum: every c_h from 1 to the capacity (32 blocks, capacity 16).
    g = torch.Generator().manual_seed(64)
    n, h = 32 * 64, 64
    q, k, v = (torch.randn(n, h, 64, generator=g).to("cuda", torch.bfloat16) for _ in range(3))
    budgets = [1 + (hh % 16) for hh in range(h)]
    mem = (torch.rand((h, 16), generator=g) * 0.3).to("cuda")
    mem_in = mem.cpu().numpy().astype(np.float64)
    idx, dem, ser = _run(ress_gpu, q, k, v, budgets, 64, 16, mem)
    _check_layer(q, k, v, 64, budgets, 16, mem_in, idx, dem, ser, mem.cpu().numpy().astype(np.float64))


def test_vasc_reset_ignores_the_memory_passed_in(ress_gpu):
    # reset = 1 starts an inference: a non-zero memory gives exactly what a
    # zeroed one gives, and is overwritten by the settled state.
    w = workloads.WORKLOADS["vggt8"]
    q, k, v = _layer_inputs(w, 0)
    pairs = ress_gpu.vasc_pairs(w.n_blocks)
    a = torch.full((w.heads, pairs), 7.0, device="cuda")
    b = torch.zeros((w.heads, pairs), device="cuda")
    ra = _run(ress_gpu, q, k, v, [50] * w.heads, w.block, 50, a, reset=True)
    rb = _run(ress_gpu, q, k, v, [50] * w.heads, w.block, 50, b, reset=False)
    for x, y in zip(ra, rb):
        assert np.array_equal(x, y)
    assert torch.equal(a, b)
