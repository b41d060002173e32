"""Builds libdynrad.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: python -m block_sparse_attention_candidate_b200.build [--force] [--verbose]
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
LIB = os.path.join(PKG, "libdynrad.so")
SOURCES = ["dynrad.cu", "host_path.cu"]
HEADERS = ["common.cuh", "candidates.cuh", "select.cuh", "attention.cuh", "sampling.cuh", "dyntok.cuh", "backward.cuh", "warp_mma.cuh",
           "optin.h"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def nvcc_command(out: str = LIB, extra=()) -> list:
    return [nvcc_path(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
            "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "--use_fast_math",
            "-I", os.path.join(ROOT, "include"),
            *extra, "-o", out] + [os.path.join(CSRC, s) for s in SOURCES]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "dynrad.h"))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force: bool = False, verbose: bool = False) -> str:
    if force or _stale():
        cmd = nvcc_command(extra=["-Xptxas", "-v"] if verbose else [])
        tmp = LIB + ".tmp"
        cmd[cmd.index("-o") + 1] = tmp
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
        if verbose:
            sys.stderr.write(r.stdout + r.stderr)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
