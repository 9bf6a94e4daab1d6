"""Build libiq8r.so in-tree: nvcc for the sm_100a kernels, g++ for the host
code, cudart linked statically so the library carries its own runtime.

    python -m quantised_fwht128_act_b200.build [--force] [--verbose]
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libiq8r.so")

CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
NVCC = os.path.join(CUDA_HOME, "bin", "nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# No fast-math anywhere: the transform and quantiser must round exactly as
# IEEE float32 (the codes are compared bit for bit).
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-ffp-contract=off",
                     f"-I{INCLUDE}", f"-I{CSRC}"]
CXX_FLAGS = ["-O2", "-std=c++17", "-fPIC", "-ffp-contract=off", "-fno-fast-math", "-Wall",
             f"-I{CUDA_HOME}/include", f"-I{INCLUDE}", f"-I{CSRC}"]

CU_SOURCES = ["iq8r_kernels.cu"]
CPP_SOURCES = ["iq8r_api.cpp", "iq8r_pack.cpp"]


def _inputs():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "iq8r.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, flush=True)
    if r.returncode != 0:
        raise RuntimeError(f"build step failed ({r.returncode}): {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    return r


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    """Compile every source and link libiq8r.so next to this file."""
    if not force and not ptxas_info and up_to_date():
        return LIB
    if not os.path.exists(NVCC):
        raise RuntimeError(f"nvcc not found at {NVCC}")
    os.makedirs(BUILD_DIR, exist_ok=True)
    objs = []
    for src in CU_SOURCES:
        obj = os.path.join(BUILD_DIR, src + ".o")
        extra = ["-Xptxas", "-v"] if ptxas_info else []
        _run([NVCC, *NVCC_FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj], verbose or ptxas_info)
        objs.append(obj)
    cxx = shutil.which("g++") or "g++"
    for src in CPP_SOURCES:
        obj = os.path.join(BUILD_DIR, src + ".o")
        _run([cxx, *CXX_FLAGS, "-c", os.path.join(CSRC, src), "-o", obj], verbose)
        objs.append(obj)
    tmp = LIB + ".tmp"
    _run([cxx, "-shared", "-o", tmp, *objs, f"-L{CUDA_HOME}/lib64", "-lcudart_static", "-lpthread", "-ldl", "-lrt",
          "-Wl,--no-undefined"], verbose)
    os.replace(tmp, LIB)
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers/spills/smem per kernel")
    args = ap.parse_args(argv)
    print(build(force=args.force, verbose=args.verbose, ptxas_info=args.ptxas_info))


if __name__ == "__main__":
    sys.exit(main())
