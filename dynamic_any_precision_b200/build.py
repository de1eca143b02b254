"""Build the in-tree shared library lib/libdpa_b200.so (sm_100a).

    python -m dynamic_any_precision_b200.build [--force] [-j N]

Decision-path sources (router, allocation) are compiled with --fmad=false and the host
encoder with -ffp-contract=off, so that every fp64 operation there is a single IEEE
round-to-nearest operation.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OUT_DIR = os.path.join(PKG, "lib")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_PATH = os.path.join(OUT_DIR, "libdpa_b200.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
               "-I", INCLUDE, "-I", CSRC] + ARCH
CU_SOURCES = {
    "route.cu": ["--fmad=false"],
    "allocate.cu": ["--fmad=false"],
    "gemv2.cu": [],
    "gemm_tc.cu": [],
    "combine.cu": [],
    "dpa_abi.cu": [],
    "route_noalloc.cu": [],
    "stack_glue.cu": [],
    "probe.cu": [],
    "rates.cu": ["--fmad=false"],
}
CPP_SOURCES = {"encode.cpp": ["-O2", "-ffp-contract=off", "-fno-fast-math"]}


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build the library")


def _headers_mtime() -> float:
    ts = [os.path.getmtime(os.path.join(INCLUDE, "dpa.h"))]
    for f in os.listdir(CSRC):
        if f.endswith((".h", ".cuh")):
            ts.append(os.path.getmtime(os.path.join(CSRC, f)))
    return max(ts)


def _compile(src: str, extra, force: bool, verbose: bool):
    path = os.path.join(CSRC, src)
    obj = os.path.join(BUILD_DIR, src + ".o")
    if not force and os.path.exists(obj):
        if os.path.getmtime(obj) >= max(os.path.getmtime(path), _headers_mtime()):
            return obj
    if src.endswith(".cu"):
        cmd = [_nvcc()] + NVCC_COMMON + extra + ["-c", path, "-o", obj]
    else:
        cmd = ["g++", "-std=c++17", "-fPIC", "-I", INCLUDE, "-I", CSRC] + extra + ["-c", path, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"compiling {src} failed:\n{res.stdout}\n{res.stderr}")
    if verbose and res.stderr.strip():
        print(res.stderr, flush=True)
    return obj


def build(force: bool = False, jobs: int = 0, verbose: bool = False) -> str:
    os.makedirs(BUILD_DIR, exist_ok=True)
    os.makedirs(OUT_DIR, exist_ok=True)
    srcs = list(CU_SOURCES.items()) + list(CPP_SOURCES.items())
    jobs = jobs or min(len(srcs), os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        objs = list(ex.map(lambda kv: _compile(kv[0], kv[1], force, verbose), srcs))
    newest = max(os.path.getmtime(o) for o in objs)
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < newest:
        cmd = [_nvcc()] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-o", LIB_PATH] + objs + ["-lpthread"]
        if verbose:
            print(" ".join(cmd), flush=True)
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"linking failed:\n{res.stdout}\n{res.stderr}")
    return LIB_PATH


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=0)
    ap.add_argument("-v", action="store_true")
    args = ap.parse_args(argv)
    print(build(args.force, args.j, args.v))
    return 0


if __name__ == "__main__":
    sys.exit(main())
