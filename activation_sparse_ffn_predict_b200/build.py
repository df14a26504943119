"""Build libasffn.so in-tree with nvcc for sm_100a (B200).

Usage: python -m activation_sparse_ffn_predict_b200.build [--force] [--ptxas-verbose]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libasffn.so")
SOURCES = [os.path.join(CSRC, "asffn.cu")]
DEPS = SOURCES + [os.path.join(CSRC, "common.cuh"), os.path.join(INCLUDE, "asffn.h")]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libasffn.so")


def command(ptxas_verbose: bool = False, out: str = LIB) -> list:
    cmd = [nvcc_path(), "-O3", "-std=c++17", "-lineinfo",
           "-gencode", "arch=compute_100a,code=sm_100a",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-shared", "-I", INCLUDE, "-I", CSRC, "-o", out] + SOURCES
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in DEPS)


def build(force: bool = False, ptxas_verbose: bool = False, quiet: bool = True) -> str:
    if not force and not ptxas_verbose and up_to_date():
        return LIB
    tmp = LIB + ".tmp"
    res = subprocess.run(command(ptxas_verbose, tmp), capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    os.replace(tmp, LIB)
    if not quiet or ptxas_verbose:
        sys.stdout.write(res.stdout + res.stderr)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, ptxas_verbose="--ptxas-verbose" in sys.argv, quiet=False)
    print(LIB)
