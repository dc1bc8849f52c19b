"""Builds libkvq.so (the CUDA kernels and the C-ABI runtime) in-tree for
sm_100a with nvcc, and with --debug libkvq_debug.so: the same sources with
KVQ_DEBUG=1, whose kernels check every index they compute against its buffer
and report a failure in the device error word (KVQ_DEVERR_SMEM / _INDEX)
instead of making the access.  kvq.py loads the debug library when the
environment has KVQ_DEBUG=1.
Usage: python -m quantized_kv_cache_14_b200.build [--force] [-v] [--debug]
(-v prints ptxas register / shared-memory usage)."""
import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libkvq.so")
BUILD = os.path.join(PKG, "_build")
LIB_DEBUG = os.path.join(PKG, "libkvq_debug.so")
BUILD_DEBUG = os.path.join(PKG, "_build_debug")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SOURCES = ["kvq_runtime.cpp", "kvq_append.cu", "kvq_decode.cu", "kvq_prefill.cu", "kvq_prefill_tc.cu", "kvq_noalloc.cu",
           "kvq_floor.cu"]
HEADERS = ["kvq_internal.h", "kvq_device.cuh", "kvq_tiles.cuh"]

FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-gencode", "arch=compute_100a,code=sm_100a",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall", "-I", os.path.join(ROOT, "include"),
         "-I", CSRC]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, verbose, debug=False):
    obj = os.path.join(BUILD_DEBUG if debug else BUILD, os.path.splitext(src)[0] + ".o")
    deps = [os.path.join(CSRC, src), os.path.join(ROOT, "include", "kvq.h")] + \
           [os.path.join(CSRC, h) for h in HEADERS]
    if not _stale(obj, deps) and not verbose:
        return obj, ""
    cmd = [NVCC] + FLAGS + (["-DKVQ_DEBUG=1"] if debug else []) + \
        (["-Xptxas", "-v"] if verbose and src.endswith(".cu") else []) + \
        ["-c", os.path.join(CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Builds libkvq.so, or libkvq_debug.so with debug=True; returns its path."""
    bdir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug else (BUILD, LIB)
    os.makedirs(bdir, exist_ok=True)
    if force:
        for f in os.listdir(bdir):
            os.remove(os.path.join(bdir, f))
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(lambda s: _compile(s, verbose, debug), SOURCES))
    objs = [o for o, _ in results]
    if verbose:
        for _, log in results:
            if log:
                print(log)
    if force or _stale(lib, objs):
        cmd = [NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs,
               "-o", lib + ".tmp", "-lcudart"]
        subprocess.check_call(cmd)
        os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
