"""Build the CUDA library in-tree: long_sequence_attention_b200/libdit_attn.so (sm_100a).

    python long_sequence_attention_b200/build.py [--force] [--verbose]

(run it by path: importing the package first would load the library it is about to replace)

One translation unit (csrc/dit_attn.cu includes every kernel), compiled by nvcc with
-gencode arch=compute_100a,code=sm_100a.  The runtime is linked statically and the driver's
cuTensorMapEncodeTiled is looked up at run time, so the library loads (and its symbols can
be inspected) on a machine without a GPU driver.  Only the dit_* symbols are exported.
"""

from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libdit_attn.so")
SRC = os.path.join(HERE, "csrc", "dit_attn.cu")
EXPORTS = os.path.join(HERE, "csrc", "exports.map")


def _sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")) + glob.glob(os.path.join(HERE, "csrc", "*.cuh"))
                  + glob.glob(os.path.join(ROOT, "include", "*.h")) + [EXPORTS])


def nvcc_command(out: str = LIB, ptxas_verbose: bool = False):
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
           "-Xlinker", f"--version-script={EXPORTS}", "-o", out, SRC]
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libdit_attn.so unless it is newer than every source file."""
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(p) for p in _sources())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = nvcc_command(tmp, ptxas_verbose=verbose)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed: " + " ".join(cmd))
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
