"""Build libprism.so (the CUDA kernels and the C ABI) in-tree for sm_100a.

    python -m dynamic_block_sparse_stats_b200.build [--jobs N] [--debug]

--debug builds libprism_debug.so instead, with -DPRISM_DEBUG: device-side
bounds checks (walk units, permutation entries) that record
PRISM_ERR_INVALID_ARG and the check's site in the workspace status word
instead of accessing out of bounds.  The binding loads it when the
environment sets PRISM_LIB=debug.

Each .cu file under csrc/ is compiled to an object with nvcc and the objects
are linked into dynamic_block_sparse_stats_b200/libprism.so.  The CUDA
runtime is linked statically and the driver API is reached through
cudaGetDriverEntryPoint, so the library loads on machines without a GPU
driver (it then fails on first use with PRISM_ERR_CUDA).
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
BUILD = os.path.join(ROOT, "_build", "prism")
LIB = os.path.join(PKG, "libprism.so")
LIB_DEBUG = os.path.join(PKG, "libprism_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found")
    return exe


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _compile(src: str, verbose: bool, debug: bool = False) -> str:
    obj = os.path.join(BUILD + ("_debug" if debug else ""), os.path.basename(src) + ".o")
    cmd = [nvcc(), *ARCH, *FLAGS, *(["-DPRISM_DEBUG"] if debug else []), "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
    if verbose and r.stderr:
        sys.stderr.write(r.stderr)
    return obj


def build(jobs: int = 4, verbose: bool = False, force: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    os.makedirs(BUILD + ("_debug" if debug else ""), exist_ok=True)
    srcs = sources()
    deps = srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    deps.append(os.path.join(ROOT, "include", "prism.h"))
    if not force and os.path.exists(lib):
        newest = max(os.path.getmtime(d) for d in deps)
        if os.path.getmtime(lib) >= newest:
            return lib
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, debug), srcs))
    cmd = [nvcc(), *ARCH, "-shared", "-o", lib + ".tmp", *objs, "-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--jobs", type=int, default=4)
    ap.add_argument("-v", "--verbose", action="store_true", help="print ptxas register/smem usage")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug", action="store_true", help="libprism_debug.so with device-side bounds checks")
    a = ap.parse_args()
    print(build(a.jobs, a.verbose, a.force, a.debug))
