"""Builds ``libmlstm_fw.so`` (all CUDA sources, sm_100a) in the package directory.

    python -m mlstm_chunkwise_b200.build [--force] [--debug-bounds]

``--debug-bounds`` builds ``libmlstm_fw_debug.so`` instead: the same sources
with ``-DMLSTM_DEBUG_BOUNDS=1``, whose kernels check the offsets of their
stores and bulk copies against the buffers' extents and report a violation in
the device error word (MLSTM_ERR_DEVICE, bit 1) instead of making the access.

nvcc cross-compiles for sm_100a without a GPU.  cudart is linked statically and
the driver API is reached through ``cudaGetDriverEntryPoint``, so the library
loads on a machine without a CUDA driver (only calls that touch a GPU fail).
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
LIB = os.path.join(PKG, "libmlstm_fw.so")
LIB_DEBUG = os.path.join(PKG, "libmlstm_fw_debug.so")
OBJDIR = os.path.join(ROOT, "_build")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
         "--expt-relaxed-constexpr"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(CSRC, "*.h"))) + sorted(glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build(debug_bounds: bool = False) -> bool:
    lib = LIB_DEBUG if debug_bounds else LIB
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _deps())


def build(force: bool = False, debug_bounds: bool = False, verbose: bool = False) -> str:
    lib = LIB_DEBUG if debug_bounds else LIB
    if not force and not needs_build(debug_bounds):
        return lib
    objdir = os.path.join(OBJDIR, "debug") if debug_bounds else OBJDIR
    os.makedirs(objdir, exist_ok=True)
    extra = ["-DMLSTM_DEBUG_BOUNDS=1"] if debug_bounds else []

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr}")
        return obj, r.stderr

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(compile_one, _sources()))
    if verbose:
        for _, err in results:
            sys.stderr.write(err)
    objs = [o for o, _ in results]
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", *objs, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc link failed:\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, debug_bounds=a.debug_bounds, verbose=a.verbose))
