"""Build libwkv7.so in-tree with nvcc for sm_100a.

Usage: ``python linear_recurrent_lm_wkv7_b200/build.py [--force] [--verbose]`` (run as a
script: importing the package loads the library, which this builds).
``--verbose`` adds ``-Xptxas -v`` (registers, spills, shared memory per kernel).
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libwkv7.so")
SOURCES = ["wkv7_api.cu", "wkv7_decode.cu", "wkv7_prefill.cu", "wkv7_prefill_pipe.cu", "wkv7_prefill_long.cu", "wkv7_gate.cu",
           "wkv7_backward.cu", "wkv7_noalloc.cu", "wkv7_state.cu"]
HEADERS = ["sm100_ptx.cuh", "wkv7_internal.cuh", "prefill_common.cuh", "tma_host.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise FileNotFoundError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "wkv7.h"), __file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not (force or verbose or _stale()):
        return LIB
    cmd = [
        nvcc_path(),
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared",
        "-I", INCLUDE,
        "-o", LIB,
    ] + [os.path.join(CSRC, f) for f in SOURCES]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
    sys.exit(0)
