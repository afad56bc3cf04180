"""Builds libfp8q.so in-tree with nvcc for sm_100a.

Usage: python -m fp4_precision_gemm_b200.build [--verbose]
Each .cu under csrc/ is compiled to an object under _build/ (only when it or a header is
newer than its object), then linked into fp4_precision_gemm_b200/libfp8q.so with the static
CUDA runtime, so the library loads on machines without a GPU (calls then return
FP8Q_ERR_CUDA).
"""
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libfp8q.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include")]
# The quantize kernels decide integer codes from FP32 arithmetic: no contraction into FMA
# (the GEMM keeps the default, its promotion uses explicit FMAs).
PER_FILE = {
    "quant_tile.cu": ["--fmad=false"],
    "quant_tensor.cu": ["--fmad=false"],
    "quant_nvfp4.cu": ["--fmad=false"],
}


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + [
        os.path.join(ROOT, "include", "fp8q.h")]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose=False, ptxas_info=False):
    os.makedirs(BUILD, exist_ok=True)
    objs = []
    hdrs = _headers()
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        name = os.path.basename(src)
        obj = os.path.join(BUILD, name.replace(".cu", ".o"))
        objs.append(obj)
        if not _stale(obj, [src] + hdrs) and not ptxas_info:
            continue
        cmd = [NVCC] + ARCH + COMMON + PER_FILE.get(name, []) + ["-c", src, "-o", obj]
        if ptxas_info:
            cmd += ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    if _stale(LIB, objs):
        cmd = [NVCC] + ARCH + ["-shared", "-o", LIB] + objs
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, ptxas_info="--ptxas-info" in sys.argv)
    print(LIB)
