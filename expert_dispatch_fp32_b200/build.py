"""Build libmoe.so in-tree with nvcc for sm_100a.

    python -m expert_dispatch_fp32_b200.build [--force] [--verbose]

Each csrc/*.cu compiles to an object under _build/ (rebuilt when it or a header
is newer), then all objects link into expert_dispatch_fp32_b200/lib/libmoe.so.
The CUDA runtime is linked statically; the driver API is reached at run time
through cudaGetDriverEntryPoint, so the library loads on hosts without a GPU.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
_BUILD = os.path.join(ROOT, "_build")
_BUILD_INSTR = os.path.join(ROOT, "_build", "instr")
LIBDIR = os.path.join(PKG, "lib")
LIB_PLAIN = os.path.join(LIBDIR, "libmoe.so")
LIB_INSTR = os.path.join(LIBDIR, "libmoe_instr.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False,
          instrument: bool = False) -> str:
    """Build libmoe.so (or, instrument=True, libmoe_instr.so: the same sources with the
    kernels' cycle counters compiled in, -DMOE_INSTRUMENT, in a build folder of its own)."""
    BUILD = _BUILD_INSTR if instrument else _BUILD
    LIB = LIB_INSTR if instrument else LIB_PLAIN
    extra = ["-DMOE_INSTRUMENT"] if instrument else []
    os.makedirs(BUILD, exist_ok=True)
    os.makedirs(LIBDIR, exist_ok=True)
    hdr_mtime = max((os.path.getmtime(h) for h in _headers()), default=0)
    objs = []
    rebuilt = False
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if (not force and os.path.exists(obj)
                and os.path.getmtime(obj) >= max(os.path.getmtime(src), hdr_mtime)):
            continue
        cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
        if ptxas_verbose:
            cmd += ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        rebuilt = True
    if rebuilt or force or not os.path.exists(LIB) or any(os.path.getmtime(o) > os.path.getmtime(LIB) for o in objs):
        tmp = LIB + ".tmp"
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    ap.add_argument("--instrument", action="store_true", help="build libmoe_instr.so (cycle counters)")
    a = ap.parse_args()
    print(build(a.force, a.verbose, a.ptxas_verbose, a.instrument))
    sys.exit(0)
