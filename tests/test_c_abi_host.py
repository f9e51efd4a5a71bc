"""The C ABI from C: tests/c_abi_check.c, a C99 program that includes
include/vdit.h and links libvdit.so, builds with gcc and its argument checks
pass.  Needs no GPU (every call it makes is rejected before CUDA is touched)."""
import os
import shutil
import subprocess

import pytest

from tests.conftest import ROOT


def test_c_program_builds_and_passes(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    import spacetime_attention_vdit_b200 as v
    if not os.path.exists(v.LIB_PATH):
        __import__("spacetime_attention_vdit_b200.build", fromlist=["build"]).build()
    libdir = os.path.dirname(v.LIB_PATH)
    exe = str(tmp_path / "c_abi_check")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi_check.c"), "-L", libdir, "-l:libvdit.so",
           "-Wl,-rpath," + libdir, "-o", exe]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
