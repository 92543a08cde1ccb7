"""Build libbkv.so (the CUDA kernels and the C ABI) for sm_100a, in-tree.

Each .cu under csrc/ is compiled by nvcc into _build/, then linked with the
static CUDA runtime into kv_cache_compression_bkv_b200/libbkv.so.  The same
sources compiled with -DBKV_DEBUG into _build_debug/ give libbkv_debug.so,
whose kernels check every data-dependent index (BKV_CHECK) and report a
failed check in the device status word instead of making the access.  nvcc
cross-compiles, so no GPU is needed to build.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libbkv.so")
BUILD_DEBUG = os.path.join(PKG, "_build_debug")
LIB_DEBUG = os.path.join(PKG, "libbkv_debug.so")
INCLUDE = os.path.join(os.path.dirname(PKG), "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
              "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newest_dep(src: str) -> float:
    deps = [src] + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps.append(os.path.join(INCLUDE, "bkv.h"))
    return max(os.path.getmtime(p) for p in deps)


def _plan(debug: bool, force: bool, extra: tuple[str, ...]):
    bdir = BUILD_DEBUG if debug else BUILD
    os.makedirs(bdir, exist_ok=True)
    flags = ["-DBKV_DEBUG"] if debug else []
    objs, cmds = [], []
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if not force and os.path.exists(obj) and os.path.getmtime(obj) >= _newest_dep(src):
            continue
        cmds.append([nvcc(), *ARCH, *NVCC_FLAGS, *flags, *extra, "-c", src, "-o", obj])
    return objs, cmds


def build(verbose: bool = False, force: bool = False, extra: tuple[str, ...] = (),
          debug: bool = True) -> str:
    """Build libbkv.so (and, with debug, libbkv_debug.so); returns libbkv.so's path."""
    variants = [(False, LIB)] + ([(True, LIB_DEBUG)] if debug else [])
    plans = [(_plan(d, force, extra), lib) for d, lib in variants]
    cmds = [c for (_, cs), _ in plans for c in cs]
    # one nvcc per translation unit, run side by side
    with ThreadPoolExecutor(max_workers=max(1, min(len(cmds), os.cpu_count() or 1))) as ex:
        for cmd in cmds:
            if verbose:
                print(" ".join(cmd), flush=True)
        for r in ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), cmds):
            if r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
                raise subprocess.CalledProcessError(r.returncode, r.args)
            if verbose and (r.stdout or r.stderr):
                print(r.stdout + r.stderr, flush=True)
    for (objs, _), lib in plans:
        if force or not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
            cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", lib, *objs]
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose=True, force="--force" in sys.argv,
          extra=tuple(a for a in sys.argv[1:] if a != "--force"))
