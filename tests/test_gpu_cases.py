"""The case runner used by the profiling commands: every case runs and leaves the device
status clean (small shapes)."""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", ["attn", "chunk", "merge", "quant", "quant_blocks", "fp8", "seg", "parts", "na3d"])
def test_case_runs(cuda_lib, case):
    cmd = [sys.executable, "-m", "long_sequence_attention_b200.cases", case, "--reps", "2",
           "--shape", "1,4,1024,128", "--grid", "2,8,16", "--window", "1,5,7"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "device status 0" in out.stdout
