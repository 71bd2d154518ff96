"""Build the CUDA library in-tree: ``lib/libmonarch_attn.so`` for sm_100a.

    python -m structured_attention_video_monarch_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libmonarch_attn.so")
MAIN = os.path.join(CSRC, "monarch_attn.cu")
BWD = os.path.join(CSRC, "monarch_bwd.cu")
HOST = os.path.join(CSRC, "monarch_host.cu")


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return (sorted(glob.glob(os.path.join(CSRC, "*.cu*")))
            + [os.path.join(ROOT, "include", "monarch_attn.h")])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources())


def nvcc_command(out: str, verbose: bool = False) -> list[str]:
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
           "-o", out, MAIN, BWD, HOST]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    return cmd


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(LIBDIR, exist_ok=True)
    tmp = LIB + f".tmp{os.getpid()}"
    proc = subprocess.run(nvcc_command(tmp, verbose), capture_output=True, text=True)
    if proc.returncode != 0:
        sys.stderr.write(proc.stdout + proc.stderr)
        raise RuntimeError("nvcc failed building libmonarch_attn.so")
    if verbose:
        sys.stderr.write(proc.stdout + proc.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
