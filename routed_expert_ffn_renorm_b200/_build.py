"""Build step: compile the CUDA sources into libmoe.so next to this file.

nvcc cross-compiles for sm_100a (B200); no GPU is needed to build.  The
CUDA runtime is linked statically so the library loads on any host with
the NVIDIA driver.  Objects go to _build/ (git-ignored); a source or flag
change rebuilds only what changed.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libmoe.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
              "-Xptxas", "-v"]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libmoe.so")
    return cand


# The bounds-checked variant (libmoe_checked.so): the same sources with
# MOE_DEBUG_BOUNDS, whose kernels range-check the index inputs a caller
# passes and report MOE_STATUS_BOUNDS instead of touching memory out of range.
VARIANTS = {"release": (LIB, BUILD_DIR, []),
            "checked": (os.path.join(HERE, "libmoe_checked.so"), os.path.join(BUILD_DIR, "checked"),
                        ["-DMOE_DEBUG_BOUNDS"])}


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(INCLUDE, "moe.h"), __file__]


def stale(variant: str = "release") -> bool:
    lib = VARIANTS[variant][0]
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force: bool = False, verbose: bool = False, variant: str = "release") -> str:
    lib, build_dir, defs = VARIANTS[variant]
    if not force and not stale(variant):
        return lib
    nvcc = _nvcc()
    os.makedirs(build_dir, exist_ok=True)
    hdr_t = max(os.path.getmtime(p) for p in _deps() if not p.endswith(".cu"))
    objs = []
    for src in sources():
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), hdr_t):
            cmd = [nvcc, *ARCH, *NVCC_FLAGS, *defs, "-I", INCLUDE, "-c", src, "-o", obj]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
                raise RuntimeError(f"nvcc failed on {os.path.basename(src)}")
            if verbose:
                sys.stderr.write(r.stderr)
        objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs, "-ldl", "-lpthread", "-lrt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"linking {os.path.basename(lib)} failed")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    variant = "checked" if "--checked" in sys.argv else "release"
    print(build(force="--force" in sys.argv, verbose=True, variant=variant))
