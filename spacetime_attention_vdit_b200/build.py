"""Build libvdit.so in place (sm_100a) with nvcc.

    python -m spacetime_attention_vdit_b200.build [--verbose-ptxas]

The library is one translation unit (csrc/vdit_api.cu includes every kernel);
the CUDA runtime is linked statically and the driver's tensor-map encoder is
looked up at run time, so the .so needs no CUDA libraries on its link line.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libvdit.so")
SOURCES = [os.path.join(CSRC, "vdit_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + [
    os.path.join(INCLUDE, "vdit.h")]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libvdit.so")


def command(ptxas_verbose: bool = False, out: str = LIB):
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC,-O2", "-shared", "-cudart", "static", "-I", INCLUDE, "-I", CSRC,
           "-o", out] + SOURCES
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile the library unless it is newer than every source; returns its path."""
    if not force and not ptxas_verbose and up_to_date():
        return LIB
    tmp = LIB + ".tmp"
    res = subprocess.run(command(ptxas_verbose, tmp), capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    os.replace(tmp, LIB)
    if ptxas_verbose:
        sys.stderr.write(res.stderr)
    return LIB


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
