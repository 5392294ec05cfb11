"""Build libcskv.so in-tree for sm_100a with nvcc.

    python compressed_sparse_kv_softmax_b200/build.py [-v] [--check]

(Run it as a script: importing it through the package would first load the
library it builds.)

Each csrc/*.cu compiles to an object under _build/ (in parallel), then the
objects link into compressed_sparse_kv_softmax_b200/libcskv.so.  With
--check (checked=True) the same sources compile with -DCSKV_CHECK under
_build_check/ into libcskv_check.so: kernels that test every index they read
from device memory and record CSKV_DEV_BOUNDS in the device status word when
one fails (the package loads it when CSKV_CHECK=1 is set in the
environment).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libcskv.so")
BUILD_CHECK = os.path.join(PKG, "_build_check")
LIB_CHECK = os.path.join(PKG, "libcskv_check.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libcskv.so")


def _compile(src: str, verbose: bool, extra, build_dir: str) -> str:
    obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
    cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, flush=True)
    return obj


def build(verbose: bool = False, extra=(), checked: bool = False) -> str:
    build_dir, lib = (BUILD_CHECK, LIB_CHECK) if checked else (BUILD, LIB)
    extra = list(extra) + (["-DCSKV_CHECK"] if checked else [])
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    with ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, extra, build_dir), srcs))
    tmp = lib + ".tmp"
    # (-ldl: the NVTX ranges look for a profiler's injection library at run time)
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-ldl"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    v = "-v" in sys.argv
    chk = "--check" in sys.argv
    extra = [a for a in sys.argv[1:] if a not in ("-v", "--check")]
    print(build(verbose=v, extra=extra, checked=chk))
