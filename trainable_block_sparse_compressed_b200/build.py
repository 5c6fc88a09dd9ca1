"""Builds libinfllmv2.so (the CUDA kernels behind the C ABI) for sm_100a.

Usage:  python -m trainable_block_sparse_compressed_b200.build [--verbose-ptxas] [--checks]

Each ``csrc/*.cu`` is compiled by nvcc into ``_build/`` at the repository
root, then linked (static CUDA runtime, no libcuda link: the driver's tensor
map encoder is fetched at run time) into ``libinfllmv2.so`` next to this file.
Objects are rebuilt only when a source or header is newer.

``--checks`` builds ``libinfllmv2_checks.so`` instead (objects in
``_build/checks``): the same kernels compiled with ``-DINFLLMV2_CHECKS``, whose
device-side index checks set INFLLMV2_STATUS_CHECK and skip the access, a
stand-in for a memory sanitizer.  The binding loads it when the environment
variable INFLLMV2_LIB names it.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libinfllmv2.so")
LIB_CHECKS = os.path.join(PKG, "libinfllmv2_checks.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
              "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in [os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"]:
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newest_dep() -> float:
    deps = glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(ROOT, "include", "infllmv2.h")]
    return max(os.path.getmtime(p) for p in deps)


def _compile(src: str, ptxas_verbose: bool, checks: bool = False) -> str:
    out_dir = os.path.join(BUILD, "checks") if checks else BUILD
    obj = os.path.join(out_dir, os.path.basename(src).replace(".cu", ".o"))
    if (os.path.exists(obj) and os.path.getmtime(obj) >= os.path.getmtime(src)
            and os.path.getmtime(obj) >= _newest_dep() and not ptxas_verbose):
        return obj
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *(["-DINFLLMV2_CHECKS"] if checks else []), "-c", src,
           "-o", obj]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
    if ptxas_verbose and r.stderr:
        sys.stderr.write(r.stderr)
    return obj


def build(ptxas_verbose: bool = False, checks: bool = False) -> str:
    lib = LIB_CHECKS if checks else LIB
    os.makedirs(os.path.join(BUILD, "checks") if checks else BUILD, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    with cf.ThreadPoolExecutor(max_workers=min(8, len(sources))) as ex:
        objs = list(ex.map(lambda s: _compile(s, ptxas_verbose, checks), sources))
    if os.path.exists(lib) and os.path.getmtime(lib) >= max(os.path.getmtime(o) for o in objs):
        return lib
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", "-cudart", "static", *objs, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--checks", action="store_true", help="build the bounds-checked library")
    args = ap.parse_args()
    print(build(args.verbose_ptxas, args.checks))
