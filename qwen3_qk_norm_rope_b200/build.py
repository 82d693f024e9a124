"""Build libqwen3attn.so in-tree for sm_100a with nvcc.

    python -m qwen3_qk_norm_rope_b200.build          # or build() from Python
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "qwen3_attn.cu")
LIB = os.path.join(PKG, "libqwen3attn.so")


def deps() -> list[str]:
    """Every source the library is built from: the .cu, its headers and the C ABI header."""
    csrc = os.path.join(PKG, "csrc")
    return sorted(os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh"))) + \
        [os.path.join(ROOT, "include", "qwen3_attn.h")]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libqwen3attn.so")


def command(out: str = LIB, ptxas_verbose: bool = False) -> list[str]:
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-o", out, SRC]
    if ptxas_verbose:
        cmd.insert(-3, "-Xptxas=-v")
    return cmd


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in deps())


def build(force: bool = False, verbose: bool = False) -> str:
    if force or not up_to_date():
        tmp = LIB + ".tmp"
        res = subprocess.run(command(tmp, ptxas_verbose=verbose), capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
        if verbose:
            sys.stderr.write(res.stdout + res.stderr)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
