"""Builds libmoe.so in-tree with nvcc for sm_100a (no GPU needed to compile).

    python -m mixture_experts_layer_27_b200.build [--debug]
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libmoe.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, debug: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    flags = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
             "-I", INCLUDE, "-I", CSRC, *ARCH]
    if debug:
        flags += ["-DMOE_DEBUG=1"]
    if verbose:
        flags += ["-Xptxas", "-v"]
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *flags, *sources(), "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, debug="--debug" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
