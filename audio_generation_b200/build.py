"""Build the sm_100a shared library libh3.so in-tree with nvcc.

Usage: python -m audio_generation_b200.build [--force]
"""

from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libh3.so")
INCLUDE = os.path.join(ROOT, "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "-shared",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [
        os.path.join(INCLUDE, "h3.h"), os.path.abspath(__file__)]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB + ".tmp"
    cmd = [nvcc] + NVCC_FLAGS + ["-I", INCLUDE, "-o", tmp] + sources()
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


def build_fault_injection(out_path: str, verbose: bool = False) -> str:
    """A test-only variant of the library (never the product build): bounded
    waits limited to 50 ms and an extra entry point, h3_test_gemm_skip_loads,
    that makes the GEMM producer issue no loads, so a test can make a wait run
    out and check the status the library reports."""
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = out_path + ".tmp"
    cmd = [nvcc] + NVCC_FLAGS + ["-DH3_FAULT_INJECTION", "-I", INCLUDE, "-o", tmp] + sources()
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, out_path)
    return out_path


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
