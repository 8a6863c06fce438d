"""Build libwan.so in-tree with nvcc for sm_100a.

    python -m video_diffusion_transformer_fwd_b200.build_lib [--force] [--debug]

The library links the CUDA runtime statically, so it loads on a machine
without a GPU (no call is made until an entry point runs). The driver entry
point it needs for TMA descriptors is fetched at run time through the
runtime, so libcuda is not a link dependency. Sources compile in parallel
(one nvcc per .cu into _build/), then link.

``debug=True`` builds libwan_debug.so with WAN_DEBUG_BOUNDS: the kernels
check every plain global store against its buffer's extent (include/wan.h,
wan_debug_bounds); load it with WAN_LIBRARY=<path>.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libwan.so")
LIB_DEBUG = os.path.join(PKG, "libwan_debug.so")
BUILD = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + [
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
    "--expt-relaxed-constexpr",
]
LINK_FLAGS = ARCH + ["-shared", "-cudart", "static"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libwan")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(lib) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force: bool = False, verbose: bool = True, debug: bool = False) -> str:
    """Compile every .cu under csrc/ into libwan.so (libwan_debug.so with
    ``debug``); skipped when up to date."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    nvcc = _nvcc()
    objdir = os.path.join(BUILD, "obj_debug" if debug else "obj")
    os.makedirs(objdir, exist_ok=True)
    flags = NVCC_FLAGS + (["-DWAN_DEBUG_BOUNDS"] if debug else [])
    jobs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        jobs.append((src, obj, [nvcc, *flags, "-I", INCLUDE, "-c", src, "-o", obj]))
    if verbose:
        print(f"nvcc {' '.join(flags)} -c <{len(jobs)} sources> -> {lib}", flush=True)
    with cf.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as ex:
        for (src, _, cmd), res in zip(jobs, ex.map(lambda j: subprocess.run(j[2], capture_output=True, text=True),
                                                   jobs)):
            if res.returncode != 0:
                sys.stderr.write(res.stdout + res.stderr)
                raise subprocess.CalledProcessError(res.returncode, cmd)
    tmp = lib + ".tmp"
    subprocess.run([nvcc, *LINK_FLAGS, "-o", tmp, *[o for _, o, _ in jobs]], check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, debug="--debug" in sys.argv)
