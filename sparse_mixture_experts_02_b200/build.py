"""Builds libmoe_b200.so and libmoe_b200_debug.so in-tree with nvcc for sm_100a (B200).

    python -m sparse_mixture_experts_02_b200.build [--force] [--verbose-ptxas] [--release-only]

Each .cu under csrc/ is compiled separately (in parallel) into _build/ (the debug build, with
-DMOE_DEBUG=1, into _build/debug/), then linked into _lib/ with the static CUDA runtime. The debug
build checks every index its kernels take from their inputs before addressing memory with it and
reports one outside its range through the status word instead of reading or writing there. The
libraries load the driver's tensor-map encoder at run time, so they do not link libcuda directly.
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
BUILD = os.path.join(PKG, "_build")
LIBDIR = os.path.join(PKG, "_lib")
LIB = os.path.join(LIBDIR, "libmoe_b200.so")
DEBUG_LIB = os.path.join(LIBDIR, "libmoe_b200_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-Wall", "--expt-relaxed-constexpr",
         "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, outdir, extra, verbose_ptxas):
    obj = os.path.join(outdir, os.path.basename(src) + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def _build_one(lib, outdir, extra, force, verbose_ptxas):
    deps = _deps()
    if not force and not verbose_ptxas and not _stale(lib, deps):
        return lib
    os.makedirs(outdir, exist_ok=True)
    os.makedirs(LIBDIR, exist_ok=True)
    srcs = _sources()
    logs = []
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        futs = [ex.submit(_compile, s, outdir, extra, verbose_ptxas) for s in srcs]
        objs = []
        for f in futs:
            o, log = f.result()
            objs.append(o)
            logs.append(log)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    if verbose_ptxas:
        sys.stderr.write("".join(logs))
    return lib


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = True) -> str:
    """Builds the release library (and, unless debug=False, the debug library); returns the
    release library's path."""
    lib = _build_one(LIB, BUILD, [], force, verbose_ptxas)
    if debug:
        _build_one(DEBUG_LIB, os.path.join(BUILD, "debug"), ["-DMOE_DEBUG=1"], force, False)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--release-only", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas, debug=not a.release_only))
