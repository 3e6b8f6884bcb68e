"""Builds libaut.so (the CUDA library behind include/aut.h) in-tree for sm_100a.

Usage: python -m audio_encoder_aut_b200.build [--force] [--verbose] [--debug-bounds]
Each source compiles to an object under _build/ (in parallel); the objects are
linked into audio_encoder_aut_b200/libaut.so with the CUDA runtime linked
statically, so the library loads on a machine without a GPU (for the host-only
planner) and needs only the driver on a GPU machine.
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
LIB = os.path.join(PKG, "libaut.so")
LIB_DEBUG = os.path.join(PKG, "libaut_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
              "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC]
SOURCES = ["aut_plan.cpp", "aut_kernels.cu", "aut_gemm.cu", "aut_attention.cu", "aut_api.cu",
           "aut_noalloc.cu", "aut_logmel.cu", "aut_inject.cu", "aut_conv1.cu"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libaut.so")


def _headers() -> list[str]:
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    return hs + [os.path.join(ROOT, "include", "aut.h")]


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, obj: str, verbose: bool, ptxas_v: bool, extra=()) -> None:
    cmd = [nvcc(), "-c", os.path.join(CSRC, src), "-o", obj] + ARCH + NVCC_FLAGS + list(extra)
    if ptxas_v and src.endswith(".cu"):
        cmd += ["-Xptxas", "-v"]
    if src.endswith(".cpp"):
        cmd += ["-x", "cu"]  # one compiler for everything; the planner has no device code
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if ptxas_v or verbose:
        sys.stdout.write(r.stdout + r.stderr)


def build(force: bool = False, verbose: bool = False, ptxas_v: bool = False,
          debug_bounds: bool = False) -> str:
    """Builds libaut.so, or with debug_bounds libaut_debug.so: the same sources
    with -DAUT_DEBUG_BOUNDS, whose kernels check their computed global
    addresses and report AUT_ERR_BOUNDS instead of trapping."""
    bdir = BUILD + ("_debug" if debug_bounds else "")
    lib_path = LIB_DEBUG if debug_bounds else LIB
    extra = ["-DAUT_DEBUG_BOUNDS"] if debug_bounds else []
    os.makedirs(bdir, exist_ok=True)
    hdrs = _headers()
    objs, jobs = [], []
    for s in SOURCES:
        obj = os.path.join(bdir, os.path.splitext(s)[0] + ".o")
        objs.append(obj)
        if force or ptxas_v or _stale(obj, [os.path.join(CSRC, s)] + hdrs):
            jobs.append((s, obj))
    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        for f in [ex.submit(_compile, s, o, verbose, ptxas_v, extra) for s, o in jobs]:
            f.result()
    LIB_ = lib_path
    if force or jobs or _stale(LIB_, objs):
        tmp = LIB_ + ".tmp"
        cmd = [nvcc(), "-shared", "-o", tmp] + objs + ARCH + ["-cudart", "static"]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB_)
    return LIB_


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print register/smem use per kernel")
    ap.add_argument("--debug-bounds", action="store_true",
                    help="build libaut_debug.so with device bounds checks instead")
    a = ap.parse_args()
    print(build(a.force, a.verbose, a.ptxas_v, a.debug_bounds))
