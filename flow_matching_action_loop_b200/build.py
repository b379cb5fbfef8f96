"""Build the action-expert shared library in-tree for sm_100a.

    python flow_matching_action_loop_b200/build.py [--force] [-v]

Compiles every csrc/*.cu and csrc/*.cpp with nvcc into _build/ and links
libflowloop.so next to this file (CUDA runtime linked statically).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libflowloop.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]
CUDA_FLAGS = ARCH + COMMON + ["--expt-relaxed-constexpr", "-Xptxas", "-v"] if os.environ.get("FR_PTXAS_V") else ARCH + COMMON + ["--expt-relaxed-constexpr"]
# FR_DEFINES="NAME ..." adds -DNAME to every compile (instrumented builds for performance analysis)
CUDA_FLAGS = CUDA_FLAGS + ["-D" + d for d in os.environ.get("FR_DEFINES", "").split()]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, verbose):
    obj = os.path.join(BUILD, os.path.basename(src) + ".o")
    flags = CUDA_FLAGS if src.endswith(".cu") else ARCH + COMMON
    cmd = [NVCC] + flags + ["-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, flush=True)
    return obj


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Build libflowloop.so, or with checked=True libflowloop_checked.so (device bounds checks,
    -DFR_DEVICE_CHECKS) in its own object directory."""
    global CUDA_FLAGS, BUILD, LIB
    if checked:
        saved = (CUDA_FLAGS, BUILD, LIB)
        CUDA_FLAGS = CUDA_FLAGS + ["-DFR_DEVICE_CHECKS"]
        BUILD = os.path.join(ROOT, "_build_checked")
        LIB = os.path.join(PKG, "libflowloop_checked.so")
        try:
            return build(force, verbose)
        finally:
            CUDA_FLAGS, BUILD, LIB = saved
    os.makedirs(BUILD, exist_ok=True)
    srcs = _sources()
    hdrs = _headers()
    objs = [os.path.join(BUILD, os.path.basename(s) + ".o") for s in srcs]
    todo = [s for s, o in zip(srcs, objs) if force or _stale(o, [s] + hdrs)]
    if todo:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(todo))) as ex:
            list(ex.map(lambda s: _compile(s, verbose), todo))
    if force or todo or _stale(LIB, objs):
        cmd = [NVCC] + ARCH + ["-shared", "-cudart", "static", "-o", LIB] + objs
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--checked", action="store_true", help="the build with device bounds checks")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose, checked=a.checked))


if __name__ == "__main__":
    sys.exit(main())
