"""Build libtpa.so in-tree with nvcc for sm_100a.

    python -m tensor_product_attention_b200.build [--verbose] [--debug]

Compiles every csrc/*.cu to an object under _build/ (parallel, skipped when up to
date) and links them with the static CUDA runtime into
tensor_product_attention_b200/libtpa.so.  Needs nvcc only, no GPU.

--debug builds the bounds-checked library libtpa_debug.so (-DTPA_DEBUG_BOUNDS, objects
under _build/debug/): every plain global access of the kernels is checked against its
buffer's extent, and a failed check records TPA_DEVERR_BOUNDS in the device error word
and skips the access.  It stands in for a memory checker on machines where none can run.
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
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libtpa.so")
DEBUG_LIB = os.path.join(PKG, "libtpa_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps(src: str) -> list[str]:
    hdrs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    return [src, os.path.join(ROOT, "include", "tpa.h")] + hdrs


def _stale(obj: str, deps: list[str]) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in deps)


def compile_one(src: str, verbose: bool, debug: bool = False) -> str:
    obj = os.path.join(BUILD, "debug" if debug else "", os.path.basename(src)[:-3] + ".o")
    if not _stale(obj, _deps(src)):
        return obj
    cmd = [nvcc()] + ARCH + FLAGS + (["-DTPA_DEBUG_BOUNDS"] if debug else []) + \
        (["-Xptxas", "-v"] if verbose else []) + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)
    return obj


def build(verbose: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    os.makedirs(os.path.join(BUILD, "debug") if debug else BUILD, exist_ok=True)
    srcs = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: compile_one(s, verbose, debug), srcs))
    if os.path.exists(lib) and all(os.path.getmtime(o) <= os.path.getmtime(lib) for o in objs):
        return lib
    tmp = lib + ".tmp"
    cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/smem usage")
    ap.add_argument("--debug", action="store_true", help="build the bounds-checked libtpa_debug.so")
    args = ap.parse_args()
    print(build(args.verbose, args.debug))


if __name__ == "__main__":
    main()
