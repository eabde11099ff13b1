"""Builds libqbsa.so in-tree with nvcc for sm_100a (static CUDA runtime, no libcuda link).

Usage: python -m quantized_block_sparse_attn_b200.build [--verbose]
"""

from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "qbsa_api.cu")
OUT = os.path.join(PKG, "libqbsa.so")
HEADERS = [os.path.join(PKG, "csrc", f) for f in os.listdir(os.path.join(PKG, "csrc"))] + [
    os.path.join(ROOT, "include", "qbsa.h")]


def nvcc_cmd(out: str = OUT, verbose: bool = False, extra=()) -> list:
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-o", out, SRC]
    if verbose:
        cmd.insert(1, "-Xptxas")
        cmd.insert(2, "-v")
    return cmd + list(extra)


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(h) <= t for h in HEADERS if os.path.isfile(h))


def build(force: bool = False, verbose: bool = False) -> str:
    if force or not up_to_date():
        cmd = nvcc_cmd(verbose=verbose)
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
        if verbose:
            sys.stdout.write(res.stdout + res.stderr)
    return OUT


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(OUT)
