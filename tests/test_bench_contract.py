"""The bench's host-side contract on the CPU: the L2 policy per workload and
the JSON line of the reference arm (the oracle timed on the host)."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from block_sparse_global_mean_b200 import workloads  # noqa: E402


def test_l2_policy_flushes_only_inputs_that_fit_twice_in_l2():
    W = workloads.WORKLOADS
    assert bench.l2_policy(W["views100"])[0] is False
    assert bench.l2_policy(W["views32"])[0] is False
    assert bench.l2_policy(W["vggt8"])[0] is True        # 69 MB of Q, K, V
    assert bench.l2_policy(W["tiny"])[0] is True
    assert "flushed" in bench.l2_policy(W["vggt8"])[1]
    assert bench.input_bytes(W["views100"]) == 3 * 140800 * 16 * 64 * 2


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "3", "--warmup", "3"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith("tiny")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
