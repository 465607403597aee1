"""Build the CUDA library ``libsvdq_b200.so`` in-tree with nvcc (sm_100a).

Usage: ``python bit_w4a4_diffusion_b200/build.py [-v]`` (or ``build()`` from
``__graft_entry__``); run it by path -- importing the package loads the
library this script produces.  Objects are rebuilt only when a source or header is
newer than the object.  Cross-compiles without a GPU.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "lib", "libsvdq_b200.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-fmad=false",
                     "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr"]
CXX_FLAGS = ["-O3", "-std=c++17", "-fPIC", "-ffp-contract=off", "-pthread", "-I", INCLUDE,
             "-I", "/usr/local/cuda/include"]

CU_SOURCES = ["abi.cu", "quantize_act.cu", "quantize_nvfp4.cu", "gemm_nvfp4.cu", "gemm_nvfp4_pair.cu", "gemm_int4.cu", "gemm_int4_pair.cu", "dequant_int4.cu", "awq_gemm.cu", "noalloc.cu"]
CXX_SOURCES = ["pack.cpp", "calib.cpp"]


def _headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    hs += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return hs


def _stale(out, deps):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"build step failed: {' '.join(cmd[:3])} ...")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)


def build(verbose=False, ptxas_verbose=False):
    """Compile every source for sm_100a and link the shared library; returns its path."""
    os.makedirs(BUILD, exist_ok=True)
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    hdrs = _headers()
    objs = []
    for src in CU_SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        objs.append(o)
        if _stale(o, [s] + hdrs) or ptxas_verbose:
            extra = ["-Xptxas", "-v"] if ptxas_verbose else []
            _run([NVCC] + NVCC_FLAGS + extra + ["-c", s, "-o", o], verbose or ptxas_verbose)
    for src in CXX_SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        objs.append(o)
        if _stale(o, [s] + hdrs):
            _run(["g++"] + CXX_FLAGS + ["-c", s, "-o", o], verbose)
    if _stale(LIB, objs):
        _run([NVCC] + ARCH + ["-shared", "-o", LIB] + objs + ["-lpthread"], verbose)
    return LIB


if __name__ == "__main__":
    build(verbose=True, ptxas_verbose="-v" in sys.argv)
