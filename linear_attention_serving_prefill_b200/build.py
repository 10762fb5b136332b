"""Builds libkda_b200.so in-tree with nvcc for sm_100a.

Usage: ``python -m linear_attention_serving_prefill_b200.build [--force]``.
Each ``csrc/*.cu`` compiles to ``_build/<name>.o`` (rebuilt when it or any
header is newer), then everything links into ``libkda_b200.so`` next to this
file, against the shared CUDA runtime so the process has one runtime instance.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libkda_b200.so")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the KDA CUDA library cannot be built")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return (glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def _compile(src: str, newest_header: float, force: bool, extra) -> str:
    obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
    if (force or not os.path.exists(obj) or os.path.getmtime(obj) < os.path.getmtime(src)
            or os.path.getmtime(obj) < newest_header):
        tmp = obj + f".tmp{os.getpid()}"
        subprocess.run([_nvcc(), *NVCC_FLAGS, *extra, "-c", src, "-o", tmp], check=True)
        os.replace(tmp, obj)
    return obj


def build(force: bool = False, extra_flags=(), jobs: int = 0) -> str:
    """Compile every csrc/*.cu for sm_100a and link libkda_b200.so; returns its path."""
    os.makedirs(BUILD, exist_ok=True)
    srcs = sources()
    newest = max([os.path.getmtime(h) for h in _headers()] + [0.0])
    with ThreadPoolExecutor(max_workers=jobs or min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, newest, force, list(extra_flags)), srcs))
    if force or not os.path.exists(LIB) or any(
            os.path.getmtime(LIB) < os.path.getmtime(o) for o in objs):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run([_nvcc(), *ARCH, "-shared", "-cudart", "shared", *objs, "-o", tmp],
                       check=True)
        os.replace(tmp, LIB)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true",
                    help="print registers / spills / shared memory per kernel")
    args = ap.parse_args()
    extra = ["-Xptxas", "-v"] if args.ptxas_verbose else []
    print(build(force=args.force or args.ptxas_verbose, extra_flags=extra))


if __name__ == "__main__":
    main()
