"""Build the CUDA library ``libkdv.so`` in-tree for sm_100a with nvcc."""
from __future__ import annotations

import concurrent.futures
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(PKG, "_build")
LIB_PATH = os.path.join(PKG, "libkdv.so")
# the same library with the verify kernel's stage stamps (include/kdv_trace.h)
TRACE_LIB_PATH = os.path.join(PKG, "libkdv_trace.so")
TRACED = "verify_tc2.cu"

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    """Compile every csrc/*.cu for sm_100a and link ``libkdv.so``. Returns its path."""
    os.makedirs(BUILD_DIR, exist_ok=True)
    headers = _headers()
    objs, jobs = [], []
    for src in _sources():
        obj = os.path.join(BUILD_DIR, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _stale(obj, [src] + headers):
            cmd = [NVCC, *ARCH, *FLAGS, *extra_flags, "-c", src, "-o", obj]
            jobs.append(cmd)

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed: {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            sys.stderr.write(r.stdout + r.stderr)

    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        list(ex.map(run, jobs))
    if force or jobs or _stale(LIB_PATH, objs):
        tmp = LIB_PATH + f".tmp{os.getpid()}"
        run([NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, "-o", tmp])
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


def build_trace(force: bool = False, verbose: bool = False) -> str:
    """Link ``libkdv_trace.so``: every object of ``libkdv.so`` except the verify
    kernel's, which is compiled again with -DKDV_TRACE. Returns its path."""
    build(force=force, verbose=verbose)
    src = os.path.join(CSRC, TRACED)
    traced_obj = os.path.join(BUILD_DIR, TRACED[:-3] + "_trace.o")
    objs = [os.path.join(BUILD_DIR, os.path.basename(s)[:-3] + ".o") for s in _sources() if not s.endswith(TRACED)]
    fresh = force or _stale(traced_obj, [src] + _headers())
    if fresh:
        cmd = [NVCC, *ARCH, *FLAGS, "-DKDV_TRACE", "-c", src, "-o", traced_obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed: {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    if fresh or _stale(TRACE_LIB_PATH, objs + [traced_obj]):
        tmp = TRACE_LIB_PATH + f".tmp{os.getpid()}"
        cmd = [NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, traced_obj, "-o", tmp]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed: {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, TRACE_LIB_PATH)
    return TRACE_LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True,
                extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []))
    if "--trace" in sys.argv:
        print(build_trace(force="--force" in sys.argv))
