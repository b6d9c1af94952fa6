"""Build libevo_attn.so (the CUDA library behind include/evo_attn.h) in-tree.

    python -m evoformer_pair_bias_b200.build [--verbose-ptxas]

Compiles the single translation unit csrc/evo_attn.cu for sm_100a with nvcc
and links it into evoformer_pair_bias_b200/libevo_attn.so.  The CUDA runtime
is linked statically; the driver API (cuTensorMapEncodeTiled) is reached
through cudaGetDriverEntryPoint, so no -lcuda is needed at link time.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "evo_attn.cu")
LIB = os.path.join(PKG, "libevo_attn.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libevo_attn.so")


def sources() -> list[str]:
    d = os.path.join(PKG, "csrc")
    return [os.path.join(d, f) for f in sorted(os.listdir(d)) if f.endswith((".cu", ".cuh"))] + [
        os.path.join(ROOT, "include", "evo_attn.h")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose_ptxas: bool = False, extra: list[str] | None = None) -> str:
    if not force and not verbose_ptxas and up_to_date():
        return LIB
    tmp = f"{LIB}.{os.getpid()}.tmp"
    cmd = [nvcc(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(PKG, "csrc"), SRC, "-o", tmp]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    if extra:
        cmd[1:1] = extra
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libevo_attn.so")
    if verbose_ptxas:
        sys.stderr.write(res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas))
