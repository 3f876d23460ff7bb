"""Build the CUDA library in-tree: ``_lib/libar_rmsnorm.so`` for sm_100a.

    python -m tensor_allreduce_residual_ar_b200.build [--force] [--ptxas-v]

Plain nvcc (no JIT, no torch extension machinery): the result is a C-ABI
shared library that any process can dlopen.  Sources are rebuilt when any of
them is newer than the library.
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
OUT = os.path.join(HERE, "_lib", "libar_rmsnorm.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile every source to an object file (in parallel, one nvcc per
    translation unit), then link the shared library."""
    if not force and up_to_date():
        return OUT
    os.makedirs(os.path.dirname(OUT), exist_ok=True)
    objdir = os.path.join(os.path.dirname(OUT), f"obj{os.getpid()}")
    os.makedirs(objdir, exist_ok=True)
    common = [_nvcc(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC",
              "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC,
              "--expt-relaxed-constexpr", "-DAR_BUILDING_LIBRARY"]
    if ptxas_verbose:
        common.insert(1, "-Xptxas=-v")
    procs, objs = [], []
    try:
        for src in sources():
            obj = os.path.join(objdir, os.path.basename(src) + ".o")
            objs.append(obj)
            procs.append((src, subprocess.Popen([*common, "-c", "-o", obj, src])))
        failed = [src for src, pr in procs if pr.wait() != 0]
        if failed:
            raise subprocess.CalledProcessError(1, f"nvcc {' '.join(failed)}")
        tmp = OUT + f".tmp{os.getpid()}"
        subprocess.run([_nvcc(), *ARCH, "-shared", "-o", tmp, *objs], check=True)
        os.replace(tmp, OUT)
    finally:
        for _, pr in procs:
            if pr.poll() is None:
                pr.kill()
        shutil.rmtree(objdir, ignore_errors=True)
    return OUT


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.ptxas_v))
    sys.exit(0)
