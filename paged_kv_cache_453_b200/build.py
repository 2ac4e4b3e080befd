"""Build libpagedkv.so in-tree with nvcc for sm_100a.

    python -m paged_kv_cache_453_b200.build [--force] [--verbose]

Compiles csrc/pagedkv.cu (all device code and the C ABI) and
csrc/allocator.cpp (host block allocator) into one shared library next to
this file. nvcc cross-compiles for sm_100a without a GPU present.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libpagedkv.so")
SOURCES = [os.path.join(CSRC, "pagedkv.cu"), os.path.join(CSRC, "allocator.cpp")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("decode.cuh", "cascade.cuh", "prefill.cuh", "prefill_tc.cuh", "prefill_tc2.cuh", "cache_ops.cuh", "ptx.cuh")] + [
    os.path.join(ROOT, "include", "pagedkv.h"), os.path.abspath(__file__)]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared",
         "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(d) > t for d in DEPS if os.path.exists(d))


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=PKG)
    os.close(fd)
    cmd = [nvcc()] + ARCH + FLAGS + SOURCES + ["-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=not verbose, text=True)
    if res.returncode != 0:
        os.unlink(tmp)
        raise RuntimeError("nvcc failed:\n" + (res.stderr or "") + (res.stdout or ""))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
