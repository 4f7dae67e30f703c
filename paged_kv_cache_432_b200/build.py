"""Builds libpagedattn.so in-tree with nvcc for sm_100a.

    python -m paged_kv_cache_432_b200.build [--verbose-ptxas] [--force]

The library is one CUDA translation unit (csrc/api.cu including the kernel
headers) plus the host-only block manager (csrc/block_manager.cpp), linked
with the static CUDA runtime so that it loads next to any PyTorch build; it
needs no libcuda at link time (the tensor-map encoder is fetched from the
driver at run time).
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libpagedattn.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(CSRC, "*.cpp")) + [os.path.join(INCLUDE, "pagedattn.h")])


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose_ptxas: bool = False, out: str = None, defines=()) -> str:
    """Compile the library (to `out`, default in-tree) if a source is newer;
    `defines` are extra -D macros (tuning variants)."""
    target = out or LIB
    if out is None and not force and not verbose_ptxas and not stale():
        return LIB
    tmp = target + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-cudart", "static", "-I", INCLUDE, "-I", CSRC,
           *[f"-D{d}" for d in defines], "-o", tmp, os.path.join(CSRC, "api.cu"),
           os.path.join(CSRC, "block_manager.cpp")]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed")
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    os.replace(tmp, target)
    return target


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas))


if __name__ == "__main__":
    main()
