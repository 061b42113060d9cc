"""Build libwkv_b200.so in-tree with nvcc for sm_100a.

    python rwkv_wkv_mixing_b200/build.py [--verbose]

No GPU is needed: nvcc cross-compiles.  The CUDA runtime is linked
statically and the driver API is reached through cudaGetDriverEntryPoint, so
the library loads on machines without a GPU driver (its calls then fail with
WKV_ERR_CUDA).
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG, "libwkv_b200.so")
SOURCES = ["capi.cu", "noalloc.cu"]
HEADERS = sorted(f for f in os.listdir(CSRC) if f.endswith(".cuh"))

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + \
        [os.path.join(INCLUDE, "wkv_b200.h"), os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, "-shared", "-I", INCLUDE, "-I", CSRC,
           *(["-Xptxas", "-v"] if verbose else []),
           "-o", tmp, *[os.path.join(CSRC, s) for s in SOURCES]]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true", help="pass -Xptxas -v")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force or a.verbose, verbose=a.verbose))


if __name__ == "__main__":
    sys.exit(main())
