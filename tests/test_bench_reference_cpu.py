"""bench.py's reference arm (the CPU oracle on bounded samples) runs without a
GPU: its one JSON line carries the keys the bench contract asks for."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"}


@pytest.mark.parametrize("workload", ["tiny", "longformer_sparse", "alibi_bias"])
def test_reference_arm_line(workload):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", workload, "--steps", "1",
                          "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert KEYS <= set(line)
    assert line["impl"] == "reference" and line["n_gpus"] == 1 and line["steps"] == 1
    assert line["value"] > 0 and line["higher_is_better"] is True and line["dtype"] == "f64"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"]
    # the same config object as our arm reports for this workload (one GPU)
    import bench
    assert line["config"] == json.loads(json.dumps(bench.config_dict(bench.StepSpec(workload, mask_tensors=False), 1)))
    if workload != "tiny":
        assert "mask" in line["config"]["workload"] or "M per head" in line["config"]["workload"]


def test_reference_arm_under_two_ranks():
    """Launched on 2 ranks, rank 0 alone runs the oracle and prints the line
    (n_gpus = 2); rank 1 exits 0 without work or output."""
    base = dict(os.environ, CUDA_VISIBLE_DEVICES="", WORLD_SIZE="2", LOCAL_RANK="0")
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "1",
           "--warmup", "3"]
    r1 = subprocess.run(cmd, cwd=ROOT, env=dict(base, RANK="1", LOCAL_RANK="1"), capture_output=True, text=True,
                        timeout=600)
    assert r1.returncode == 0, r1.stderr[-2000:]
    assert r1.stdout.strip() == ""
    r0 = subprocess.run(cmd, cwd=ROOT, env=dict(base, RANK="0"), capture_output=True, text=True, timeout=600)
    assert r0.returncode == 0, r0.stderr[-2000:]
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
