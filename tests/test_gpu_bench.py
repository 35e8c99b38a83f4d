"""bench.py's output contract on a B200 (tiny workload, a few steps)."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def test_bench_json_line_contract():
    cmd = [sys.executable, "bench.py", "--workload", "tiny", "--steps", "5", "--warmup", "3", "--cpu-seconds", "0.5"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(l) for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = lines[0]
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "clocks", "e2e",
                "gpu_launches"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 5 and d["warmup"] == 3 and d["value"] > 0
    assert d["config"]["workload"] == "tiny" and d["device_status"] == 0
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["achieved"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-4          # frac is rounded to 4 places
    assert d["e2e"]["h2d_bytes_per_step"] == 3 * 2 * 256 * 64 * 2 and d["e2e"]["d2h_bytes_per_step"] > 0
    assert d["e2e"]["head_groups"] == 1 and d["e2e"]["matches_whole_tensor_calls"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["gpu_launches"] == 5 * 4                        # fwd + 2 chunks + merge per step
    assert d["merge_roofline"]["bound"] == "hbm"
    assert d["clocks"]["samples"] >= 1 and d["clocks"]["sm_mhz"] > 0
    f = d["forwards"]
    for key in ("sd3_1024_bf16", "flux_1024_bf16", "flux_2048_bf16", "video_bf16", "flux_2048_e4m3", "video_e4m3"):
        assert f[key]["tflops"] > 0 and 0 < f[key]["frac"] < 2, (key, f[key])


def test_bench_video_e2e_pipeline_matches():
    """Video workload (bf16 + e4m3 variant): the head-group pipeline of the end-to-end leg
    reproduces the whole-tensor calls bit for bit."""
    cmd = [sys.executable, "bench.py", "--workload", "video", "--steps", "3", "--warmup", "3",
           "--skip-cpu-baseline", "--e2e-groups", "5"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    d = [json.loads(l) for l in out.stdout.splitlines() if l.startswith("{")][0]
    assert d["e2e"]["head_groups"] == 5 and d["e2e"]["matches_whole_tensor_calls"] is True
    assert d["device_status"] == 0


@pytest.mark.parametrize("mode", ["ring", "ring_peers", "ulysses", "ulysses_peers"])
def test_bench_sequence_parallel_modes_on_one_gpu(mode):
    """bench.py --mode <form> on one rank (a one-rank NCCL group): the JSON contract, strong
    scaling, and the rank's rows agreeing with a single launch over the whole sequence."""
    cmd = [sys.executable, "bench.py", "--mode", mode, "--workload", "sd3_1024", "--steps", "3", "--warmup", "3",
           "--skip-cpu-baseline"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(l) for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = lines[0]
    assert d["scaling"] == "strong" and d["config"]["parallelism"] == mode + "1" and d["value"] > 0
    assert d["device_status"] == 0 and d["gpu_launches"] > 0
    assert d["max_abs_vs_single_launch"] <= 2e-2 and d["lse_max_abs_vs_single_launch"] <= 1e-3
    assert d["e2e"]["h2d_bytes_per_step"] == 3 * 2 * 24 * 4429 * 64 * 2
