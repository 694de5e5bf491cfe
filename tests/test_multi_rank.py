"""Host-side logic of the multi-GPU run on the CPU with the gloo backend and
two ranks: every rank draws its own input, timings are reduced as the maximum
over ranks, and the whole-job value counts the units of all ranks."""

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
