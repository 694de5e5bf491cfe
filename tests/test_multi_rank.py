"""Host-side logic of the multi-GPU run on the CPU with the gloo backend and
two ranks: every rank draws its own input, timings are reduced as the maximum
over ranks, and the whole-job value counts the units of all ranks; with the
head split, each rank computes its heads of one input (the oracle stands in
for the kernels) and the gathered result equals the unsharded one."""

import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_global_mean_b200 import workloads
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = workloads.scaled(workloads.WORKLOADS["vggt8"], 1)
        qx, _, _ = workloads.generate(w, seed=bench.rank_seed(w, rank))
        digest = float(qx.float().sum())
        # rank r "took" 10 + 5 r ms and 100 + r ms
        got = bench.max_over_ranks([10.0 + 5 * rank, 100.0 + rank], "cpu", world)
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        q.put((rank, got, digests))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_draw_distinct_inputs():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, digests in results:
        assert got == [15.0, 101.0]
        assert digests[0] != digests[1]


def test_whole_job_value_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_tflops(8e12, 10, 1, 100.0)
    two = bench.whole_job_tflops(8e12, 10, 2, 100.0)
    assert one == pytest.approx(800.0)
    assert two == pytest.approx(2 * one)


def test_reference_arm_exits_quietly_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def _head_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    import oracle
    from block_sparse_global_mean_b200 import workloads
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = workloads.scaled(workloads.WORKLOADS["vggt8"], 1, name="split")   # 1,408 tokens, H=16
        full = workloads.generate(w)
        h0, h1 = bench.head_slice(w.heads, world, rank)
        qs, ks, vs = (t.double().numpy() for t in bench.shard_heads(full, h0, h1))
        assert qs.flags["C_CONTIGUOUS"] and qs.shape[1] == h1 - h0
        idx = oracle.select_blocks(qs, ks, None, w.block, w.budget)
        rows = [(h, i) for h in range(h1 - h0) for i in (0, w.n_blocks - 1)]
        out, lse = oracle.sparse_attention(qs, ks, vs, idx, w.block, rows=rows)
        parts = [None] * world
        dist.all_gather_object(parts, (h0, h1, idx, out, lse))
        if rank == 0:
            qf, kf, vf = (t.double().numpy() for t in full)
            ref_idx = oracle.select_blocks(qf, kf, None, w.block, w.budget)
            ok = True
            for a, b, idx_r, out_r, lse_r in parts:
                ok &= np.array_equal(idx_r, ref_idx[a:b])
                rows_f = [(a + h, i) for h in range(b - a) for i in (0, w.n_blocks - 1)]
                ref_o, ref_l = oracle.sparse_attention(qf, kf, vf, ref_idx, w.block, rows=rows_f)
                ok &= np.allclose(out_r, ref_o[:, a:b], equal_nan=True, atol=1e-12)
                ok &= np.allclose(lse_r, ref_l[a:b], equal_nan=True, atol=1e-12)
            covered = sorted(h for a, b, *_ in parts for h in range(a, b))
            q.put((ok, covered))
    finally:
        dist.destroy_process_group()


def test_head_split_over_two_gloo_ranks_equals_the_unsharded_result():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_head_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    ok, covered = q.get(timeout=300)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert ok
    assert covered == list(range(16))


def test_head_slice_rejects_uneven_splits():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.head_slice(16, 4, 3) == (12, 16)
    with pytest.raises(ValueError):
        bench.head_slice(16, 3, 0)


def _vasc_head_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    import oracle
    from block_sparse_global_mean_b200 import workloads
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = workloads.scaled(workloads.WORKLOADS["vggt8"], 1, name="split")   # 22 blocks, H=16
        budgets = [3 + (h % 7) for h in range(w.heads)]
        h0, h1 = bench.head_slice(w.heads, world, rank)
        mem = None
        mine = []
        for layer in range(2):
            full = workloads.generate(w, seed=w.seed + 1000 * (layer + 1))
            qs, ks, vs = (t.double().numpy() for t in bench.shard_heads(full, h0, h1))
            idx, mem, _ = oracle.select_blocks_vasc(qs, ks, vs, w.block, budgets[h0:h1], 9, mem)
            mine.append((idx, mem))
        parts = [None] * world
        dist.all_gather_object(parts, (h0, h1, mine))
        if rank == 0:
            ok = True
            ref_mem = None
            for layer in range(2):
                full = workloads.generate(w, seed=w.seed + 1000 * (layer + 1))
                qf, kf, vf = (t.double().numpy() for t in full)
                ref_idx, ref_mem, _ = oracle.select_blocks_vasc(qf, kf, vf, w.block, budgets, 9,
                                                                ref_mem)
                for a, b, rmine in parts:
                    ok &= np.array_equal(rmine[layer][0], ref_idx[a:b])
                    ok &= np.allclose(rmine[layer][1], ref_mem[a:b], rtol=0, atol=1e-15)
            q.put(ok)
    finally:
        dist.destroy_process_group()


def test_vasc_head_split_over_two_gloo_ranks_equals_the_unsharded_layers():
    """The VASC layer shards by head: each rank keeps its heads' memory, and
    two layers on two ranks give the kept sets and memory of the unsharded
    run (the memory copy is normalised per head, budgets are per head)."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_vasc_head_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    ok = q.get(timeout=300)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert ok
