"""Benchmark of the block-sparse global-attention hot path on B200.

One step = one pass of the hot path over one synthetic multi-view input:
pooled block selection (pool + pooled scores + exact top-k) followed by the
block-sparse attention forward; with --workload views200 the step also runs
the drift stage.  Default workload: 100 views x 1,408 tokens (N = 140,800),
H = 16, d = 64, block 64, 220 of 2,200 key blocks kept (90 % sparsity).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

With N > 1 launch one process per GPU with torch.distributed.run; every rank
processes its own input (weak scaling, no data-path collective) and rank 0
prints one JSON line.  `--impl reference` times the CPU oracle instead (rank 0
only), on bounded samples of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_global_mean_b200 import workloads  # noqa: E402

METRIC = "block-sparse attn effective TFLOPS & % bf16 peak at 90% sparsity; speedup vs dense"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["ress_attn.cu", "ress_common.cuh"]


def input_bytes(w) -> int:
    """Q + K + V bytes one step reads."""
    elem = 2 if w.dtype == "bf16" else 4
    return 3 * w.n_tokens * w.heads * w.head_dim * elem


def l2_policy(w):
    """(flush, description): inputs under twice the L2 size are timed with an
    L2 flush (a 256 MB write) before every timed step, outside its events."""
    mb = input_bytes(w) / 1e6
    if input_bytes(w) >= 2 * L2_BYTES:
        return False, "inputs larger than L2 (Q+K+V = %.0f MB per step)" % mb
    return True, "L2 flushed before every timed step by a 256 MB write outside the timed events " \
                 "(Q+K+V = %.1f MB per step)" % mb


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_hash(names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "block_sparse_global_mean_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per attention launch from a committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"attn_{workload}_dram.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_sha") != kernel_hash(KERNEL_SOURCES):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.index = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="views100", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-dense", action="store_true", help="skip the dense SDPA comparison")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end pass")
    return ap.parse_args()


def rank_seed(w, rank: int) -> int:
    """Every rank draws its own input (weak scaling over independent inputs)."""
    return w.seed + 1000 * rank


def max_over_ranks(values, device, world: int):
    """Element-wise maximum of per-rank timings (a collective when world > 1)."""
    t = torch.tensor(values, device=device, dtype=torch.float64)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def whole_job_tflops(flops_per_step: float, steps: int, world: int, max_elapsed_ms: float) -> float:
    """Units processed by all ranks divided by the slowest rank's time."""
    return flops_per_step * steps * world / (max_elapsed_ms / 1e3) / 1e12


def workload_config(w, world: int):
    return {
        "workload": (f"{w.name}: {w.views} views x {w.tokens_per_view} tokens (N={w.n_tokens}), "
                     f"H={w.heads}, d={w.head_dim}, block {w.block}, budget {w.budget} of "
                     f"{w.n_blocks} ({100 * w.sparsity:.0f}% sparsity), lambda {w.lam}"),
        "global_batch": world,
        "tokens_per_rank": w.n_tokens,
        "step": "select(pool+score+topk) -> block-sparse attention" + (" -> drift" if w.drift else ""),
        "l2": l2_policy(w)[1],
        "parallelism": f"dp{world} (independent inputs per rank)",
    }


# --------------------------------------------------------------------------
# CPU oracle timing (the reported baseline)
# --------------------------------------------------------------------------

def cpu_oracle_rate(w, q_cpu, k_cpu, v_cpu, seconds_target: float = 12.0):
    """Times the CPU oracle on a bounded sample of one step and extrapolates to
    the full step.  Returns (TFLOPS, sample description, threads)."""
    import numpy as np

    import oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        threads = os.cpu_count() or 1
    h0 = 0
    qh = q_cpu[:, h0:h0 + 1].double().numpy()
    kh = k_cpu[:, h0:h0 + 1].double().numpy()
    vh = v_cpu[:, h0:h0 + 1].double().numpy()
    t0 = time.perf_counter()
    idx_h = oracle.select_blocks(qh, kh, vh if w.lam else None, w.block, w.budget, w.lam)
    t_sel_head = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    rows = 0
    t_rows = 0.0
    while t_rows < seconds_target and rows < 256:
        i = int(rng.integers(w.n_blocks))
        t0 = time.perf_counter()
        o, lse = oracle.sparse_attention_block(qh, kh, vh, idx_h[0, i], 0, i, w.block)
        if w.drift:
            oracle.drift_block(qh, kh, vh, idx_h[0, i], lse, 0, i, w.block)
        t_rows += time.perf_counter() - t0
        rows += 1
    t_step = t_sel_head * w.heads + (t_rows / rows) * (w.heads * w.n_blocks)
    tflops = w.effective_flops() / t_step / 1e12
    sample = (f"selection of head 0 (all {w.n_blocks} query blocks) and {rows} attention rows"
              f"{' + drift' if w.drift else ''} of head 0, extrapolated to the full step "
              f"({w.heads} heads x {w.n_blocks} query blocks): {t_step:.1f} s per step")
    return tflops, sample, threads


# --------------------------------------------------------------------------
# Reference arm: the CPU oracle
# --------------------------------------------------------------------------

def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    w = workloads.WORKLOADS[args.workload]
    q, k, v = workloads.generate(w)
    rates = []
    samples = ""
    threads = 1
    for s in range(args.warmup + args.steps):
        rate, samples, threads = cpu_oracle_rate(w, q, k, v, seconds_target=2.0)
        if s >= args.warmup:
            rates.append(rate)
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": w.effective_flops() / (value * 1e12) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, 1),
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
                         "sample": samples},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# Our arm
# --------------------------------------------------------------------------

def run_ours(args, rank: int, world: int, local_rank: int):
    import torch.distributed as dist

    from block_sparse_global_mean_b200 import ress

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.WORKLOADS[args.workload]
    peaks, peak_kind = load_peaks()
    q_cpu, k_cpu, v_cpu = workloads.generate(w, seed=rank_seed(w, rank))
    q, k, v = (t.to(dev) for t in (q_cpu, k_cpu, v_cpu))
    stream = torch.cuda.current_stream(dev)
    nb, H, B = w.n_blocks, w.heads, w.block
    lam = w.lam
    idx = torch.empty((H, nb, w.budget), dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((H, w.n_tokens), dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, ress.select_workspace_bytes(w.n_tokens, H, B, q.dtype, lam)),
                     dtype=torch.uint8, device=dev)
    drift = set_drift = None
    if w.drift:
        drift = torch.empty((H, nb, nb - w.budget), dtype=torch.float32, device=dev)
        set_drift = torch.empty((H, nb), dtype=torch.float32, device=dev)
    launches_per_step = (3 if lam else 2) + 1 + (1 if w.drift else 0)

    ev = {n: [] for n in ("sel0", "sel1", "att0", "att1", "dr0", "dr1")}

    def step(qq, kk, vv, record=False):
        if record:
            e = torch.cuda.Event(enable_timing=True); e.record(stream); ev["sel0"].append(e)
        ress.ress_select_blocks(qq, kk, vv if lam else None, w.budget, lam, B, idx=idx, workspace=ws,
                                stream=stream)
        if record:
            e = torch.cuda.Event(enable_timing=True); e.record(stream); ev["sel1"].append(e)
            e = torch.cuda.Event(enable_timing=True); e.record(stream); ev["att0"].append(e)
        ress.ress_block_sparse_attn(qq, kk, vv, idx, B, out=out, lse=lse, stream=stream)
        if record:
            e = torch.cuda.Event(enable_timing=True); e.record(stream); ev["att1"].append(e)
        if w.drift:
            if record:
                e = torch.cuda.Event(enable_timing=True); e.record(stream); ev["dr0"].append(e)
            ress.ress_block_drift(qq, kk, vv, idx, lse, B, drift=drift, set_drift=set_drift,
                                  stream=stream)
            if record:
                e = torch.cuda.Event(enable_timing=True); e.record(stream); ev["dr1"].append(e)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    for _ in range(args.warmup):
        step(q, k, v)
    torch.cuda.synchronize(dev)
    status, detail = ress.ress_check_device_errors(stream, dev)
    if status != 0:
        raise RuntimeError(f"device error {status} (detail {detail}) during warm-up")

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    flush, _ = l2_policy(w)
    scratch = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush else None
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for it in range(args.steps):
        if flush:
            scratch.fill_(it & 255)
        step(q, k, v, record=True)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    if flush:
        # Each step from its first to its last event; the flushes lie between.
        last = ev["dr1"] if w.drift else ev["att1"]
        elapsed_ms = sum(a.elapsed_time(b) for a, b in zip(ev["sel0"], last))
    else:
        elapsed_ms = t_start.elapsed_time(t_end)

    def mean_pair(a, b):
        return sum(x.elapsed_time(y) for x, y in zip(ev[a], ev[b])) / max(1, len(ev[a]))

    sel_ms = mean_pair("sel0", "sel1")
    att_ms = mean_pair("att0", "att1")
    dr_ms = mean_pair("dr0", "dr1") if w.drift else None

    # End to end through the public API with host buffers: H2D of Q, K, V from
    # pinned memory, the step, D2H of the output.
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (t.pin_memory() for t in (q_cpu, k_cpu, v_cpu))
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

        def e2e_step():
            qd.copy_(qh, non_blocking=True)
            kd.copy_(kh, non_blocking=True)
            vd.copy_(vh, non_blocking=True)
            step(qd, kd, vd)
            out_h.copy_(out, non_blocking=True)

        for _ in range(max(1, args.warmup // 2)):
            e2e_step()
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_ms = e0.elapsed_time(e1)
        h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
        d2h = out_h.numel() * out_h.element_size()
        e2e = {"ms": e2e_ms, "h2d": h2d, "d2h": d2h}
    clock_info = clocks.stop()

    status, detail = ress.ress_check_device_errors(stream, dev)
    if status != 0:
        raise RuntimeError(f"device error {status} (detail {detail}) in the timed region")

    elapsed_ms, e2e_ms = max_over_ranks([elapsed_ms, e2e["ms"] if e2e else 0.0], dev, world)

    # Dense SDPA on the same shapes (fastest backend), for the speedup.
    dense = None
    if not args.no_dense and rank == 0:
        dense = dense_baseline(q, k, v, stream)

    if rank != 0:
        return
    flops = w.effective_flops()
    value = whole_job_tflops(flops, args.steps, world, elapsed_ms)
    att_tflops = flops / (att_ms / 1e3) / 1e12
    peak_tf = float(peaks["bf16_tflops"])
    peak_tf_sus = float(peaks.get("bf16_tflops_sustained", peak_tf))
    sel_bytes = 2 * w.n_tokens * H * 64 * 2 + H * nb * w.budget * 4
    if lam:
        sel_bytes += w.n_tokens * H * 64 * 2
    sel_gbs = sel_bytes / (sel_ms / 1e3) / 1e9
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded clustered multi-view tokens; no dataset or weights)",
        "config": workload_config(w, world),
        "roofline": {
            "kernel": "block_sparse_attn_kernel",
            "bound": "tensor",
            "achieved": att_tflops,
            "peak": peak_tf,
            "unit": "TFLOP/s",
            "frac": att_tflops / peak_tf,
            "peak_kind": f"{peak_kind} bf16 burst",
            "frac_of_sustained": att_tflops / peak_tf_sus,
            "traffic": recorded_traffic(w.name),
            "algorithmic": "4*N*kept_keys*d*H = %.4g FLOP per launch" % flops,
        },
        "stages": {
            "select_ms": sel_ms,
            "select_gbs": sel_gbs,
            "select_hbm_frac": sel_gbs / float(peaks["hbm_gbs"]),
            "select_bytes": sel_bytes,
            "attn_ms": att_ms,
            "attn_tflops": att_tflops,
        },
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clock_info,
    }
    if w.drift:
        line["stages"]["drift_ms"] = dr_ms
        line["stages"]["drift_tflops"] = w.drift_flops() / (dr_ms / 1e3) / 1e12
    if dense:
        line["dense"] = dense
        line["dense"]["speedup_vs_sparse_attn"] = dense["ms"] / att_ms
        line["dense"]["speedup_vs_step"] = dense["ms"] / (elapsed_ms / args.steps)
    if e2e:
        line["e2e"] = {"value": whole_job_tflops(flops, args.steps, world, e2e_ms), "unit": "TFLOPS",
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                       "ms_per_step": e2e_ms / args.steps}
    if world == 1 and not args.no_cpu:
        rate, sample, threads = cpu_oracle_rate(w, q_cpu, k_cpu, v_cpu)
        line["cpu_baseline"] = {"value": rate, "unit": "TFLOPS", "cores": threads,
                                "kind": "oracle", "sample": sample}
    print(json.dumps(line), flush=True)


def dense_baseline(q, k, v, stream):
    """Fastest torch SDPA backend for dense attention on the same shapes."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    import torch.nn.functional as F

    qt, kt, vt = (t.unsqueeze(0).transpose(1, 2) for t in (q, k, v))   # [1, H, N, d] views
    best = None
    for name, be in (("flash", SDPBackend.FLASH_ATTENTION), ("cudnn", SDPBackend.CUDNN_ATTENTION),
                     ("efficient", SDPBackend.EFFICIENT_ATTENTION)):
        try:
            with sdpa_kernel([be]):
                F.scaled_dot_product_attention(qt, kt, vt)
                torch.cuda.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                reps = 3
                for _ in range(reps):
                    F.scaled_dot_product_attention(qt, kt, vt)
                e1.record(stream)
                torch.cuda.synchronize()
                ms = e0.elapsed_time(e1) / reps
        except Exception:  # noqa: BLE001 - a backend may not support the shape
            continue
        if best is None or ms < best["ms"]:
            best = {"backend": name, "ms": ms}
    if best:
        n, h = q.shape[0], q.shape[1]
        best["tflops"] = 4.0 * n * n * 64 * h / (best["ms"] / 1e3) / 1e12
    return best


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
