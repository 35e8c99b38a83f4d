"""The library used from plain C: tests/c/abi_from_c.c includes include/dit_attn.h, links
libdit_attn.so with gcc and checks version, status strings and argument validation (no GPU
involved: every attention call carries an invalid argument)."""

import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_c_program_links_and_validates(tmp_path):
    import __graft_entry__
    __graft_entry__._build_module().build()
    libdir = os.path.join(ROOT, "long_sequence_attention_b200")
    exe = str(tmp_path / "abi_from_c")
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                         os.path.join(ROOT, "tests", "c", "abi_from_c.c"), "-L", libdir, "-l:libdit_attn.so",
                         f"-Wl,-rpath,{libdir}", "-o", exe], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "abi_from_c ok" in run.stdout
