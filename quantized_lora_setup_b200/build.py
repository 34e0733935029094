"""Build libaqnf4.so (the C-ABI library) in-tree for sm_100a with nvcc.

``python -m quantized_lora_setup_b200.build`` or ``build()``; the shared library lands in
``quantized_lora_setup_b200/lib/libaqnf4.so``.  No fast-math and no implicit FMA
contraction: the kernels rely on IEEE rounding, exactly as written, for bit-exact NF4 codes.
"""
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIB_DIR, "libaqnf4.so")
SOURCES = ["codebook.cpp", "quant_score.cu", "double_quant.cu", "dequant.cu", "select.cu",
           "selftest.cu", "nf4_gemm.cu"]
HEADERS = ["internal.h", "device.cuh"]

# -fmad=false: no multiply and add is ever fused behind the code's back (every FMA the
# kernels want is written out).  A fused x*r - mid decides ties against the exact product
# instead of the rounded v = fl(x*r) and flips codes where v equals a midpoint exactly.
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-fmad=false",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--shared", "-cudart", "static",
]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: cannot build libaqnf4")


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "aqnf4.h"))
    return files


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    """Compile libaqnf4.so if it is missing or older than a source; return its path."""
    newest = max(os.path.getmtime(f) for f in _inputs())
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, *extra_flags, "-I", INCLUDE, "-I", CSRC, "-o", tmp,
           *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True,
                extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else ()))
