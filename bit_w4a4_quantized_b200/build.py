"""Build libsvdq.so in-tree: CUDA kernels for sm_100a (nvcc) + host C++ (g++).

Usage: ``python -m bit_w4a4_quantized_b200.build [--force] [-v]``.  Object
files go to ``bit_w4a4_quantized_b200/_build``; the library to
``bit_w4a4_quantized_b200/libsvdq.so``.  Rebuilds only when a source or header
is newer than the library.
"""

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libsvdq.so")

CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
NVCC = os.path.join(CUDA_HOME, "bin", "nvcc")

CU_SOURCES = ["act_quant.cu", "gemm.cu", "lora.cu", "mlp_static.cu", "w4a16.cu"]
CPP_SOURCES = ["api.cpp", "blob.cpp", "prepare.cpp", "svd.cpp"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-I" + INCLUDE,
]
# prepare.cpp takes the quantization decisions: no FMA contraction there.
CXX_FLAGS = ["-O3", "-std=c++17", "-fPIC", "-fvisibility=hidden", "-march=x86-64-v3", "-pthread",
             "-I" + INCLUDE, "-I" + os.path.join(CUDA_HOME, "include")]
CXX_EXTRA = {"prepare.cpp": ["-ffp-contract=off"], "api.cpp": ["-ffp-contract=off"]}


def _sources():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "svdq.h"))
    files.append(os.path.abspath(__file__))
    return files


def needs_build():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _sources())


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"build step failed: {' '.join(cmd[:3])} ... ({r.returncode})")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)
    return r


def build(force=False, verbose=False, ptxas_verbose=False):
    """Compile every source and link libsvdq.so; returns the library path."""
    if not force and not needs_build():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    objs = []
    for f in CU_SOURCES:
        o = os.path.join(BUILD, f + ".o")
        extra = ["-Xptxas", "-v"] if ptxas_verbose else []
        _run([NVCC, *NVCC_FLAGS, *extra, "-c", os.path.join(CSRC, f), "-o", o], verbose or ptxas_verbose)
        objs.append(o)
    cxx = shutil.which("g++") or "g++"
    for f in CPP_SOURCES:
        o = os.path.join(BUILD, f + ".o")
        _run([cxx, *CXX_FLAGS, *CXX_EXTRA.get(f, []), "-c", os.path.join(CSRC, f), "-o", o], verbose)
        objs.append(o)
    tmp = LIB + ".tmp"
    _run([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp, *objs,
          "-Xcompiler", "-pthread", "-lrt", "-ldl"], verbose)
    os.replace(tmp, LIB)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_verbose=a.ptxas_verbose))


if __name__ == "__main__":
    main()
