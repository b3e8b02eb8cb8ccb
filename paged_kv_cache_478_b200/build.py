"""Build libpagedattn.so in-tree with nvcc for sm_100a.

    python -m paged_kv_cache_478_b200.build [--force] [--verbose]

The library is written next to this file so that it travels with the source
tree; the Python binding loads it from there and nowhere else.
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libpagedattn.so")
BUILD_DIR = os.path.join(ROOT, "_build")

CU_SOURCES = ["pagedattn.cu"]
CPP_SOURCES = ["block_manager.cpp", "status.cpp"]
HEADERS = ["device_utils.cuh", "plan.cuh", "decode.cuh", "cache_ops.cuh", "status.h", "mma_utils.cuh",
           "shared_prefix.cuh", "decode_gqa.cuh", "prefill.cuh", "tma.cuh"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _inputs():
    files = [os.path.join(CSRC, f) for f in CU_SOURCES + CPP_SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "pagedattn.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    objs = []
    common = ["-O3", "-std=c++17", "-I", INCLUDE, "-I", CSRC]
    for src in CU_SOURCES:
        obj = os.path.join(BUILD_DIR, src + ".o")
        cmd = [NVCC, *ARCH, "-lineinfo", *common, "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
               "-c", os.path.join(CSRC, src), "-o", obj]
        if ptxas_verbose:
            cmd.insert(1, "-Xptxas=-v")
        _run(cmd, verbose)
        objs.append(obj)
    for src in CPP_SOURCES:
        obj = os.path.join(BUILD_DIR, src + ".o")
        _run(["g++", *common, "-fPIC", "-Wall", "-c", os.path.join(CSRC, src), "-o", obj], verbose)
        objs.append(obj)
    tmp = LIB + f".tmp{os.getpid()}"
    _run([NVCC, *ARCH, "-shared", "-cudart", "static", *objs, "-o", tmp], verbose)
    os.replace(tmp, LIB)
    return LIB


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or r.returncode != 0:
        sys.stdout.write(r.stdout)
        sys.stderr.write(r.stderr)
    if r.returncode != 0:
        raise RuntimeError(f"build step failed: {' '.join(cmd)}")


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, ptxas_verbose=args.ptxas_verbose))
