"""Builds libsvdq_b200.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: python -m bit_w4a4_diffusion_smooth_b200.build_lib [--force]

Objects go to bit_w4a4_diffusion_smooth_b200/_build/, the shared library next
to this file.  Translation units are compiled in parallel; a unit is rebuilt
when it or any header under csrc/ or include/ is newer than its object.
"""
import argparse
import concurrent.futures
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libsvdq_b200.so")

SOURCES = ["api.cu", "quant_act.cu", "act_amax.cu", "gemm_w4a4.cu", "gemm_w4a4_requant.cu", "gemv_w4a16.cu",
           "awq_gemm.cu", "int4_gemm.cu", "int4_gemm_tc.cu", "pack_svdq.cpp", "pack_awq.cpp", "pack_int4.cpp", "pack_device.cu"]
# The device pack's float64 products and the many-row AWQ GEMM run on cuBLAS / cuBLASLt (plain GEMMs); the
# toolkit's copies are found through the rpath.
CUDA_LIB = os.path.join(os.path.dirname(os.path.dirname(shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc")), "lib64")
LINK_LIBS = ["-lpthread", "-lcublas", "-lcublasLt", "-Xlinker", f"-rpath={CUDA_LIB}"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# Host code: no fused multiply-add contraction and no fast-math, so the
# float32 quantization decisions of the host pack follow IEEE one rounding per
# operation.
HOST_FLAGS = ["-Xcompiler", "-fPIC,-O3,-ffp-contract=off,-fno-fast-math,-pthread"]
COMMON = ["-std=c++17", "-O3", "-lineinfo", "-I", INCLUDE, "-I", CSRC] + HOST_FLAGS


def nvcc():
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build the library")
    return path


def _headers_mtime():
    newest = 0.0
    for d in (CSRC, INCLUDE):
        for f in os.listdir(d):
            if f.endswith((".h", ".cuh", ".hpp")):
                newest = max(newest, os.path.getmtime(os.path.join(d, f)))
    return newest


def _compile(src, force, verbose):
    obj = os.path.join(BUILD, src + ".o")
    path = os.path.join(CSRC, src)
    if (not force and os.path.exists(obj)
            and os.path.getmtime(obj) >= max(os.path.getmtime(path), _headers_mtime())):
        return obj, ""
    cmd = [nvcc()] + COMMON + ARCH + ["-c", path, "-o", obj]
    if src.endswith(".cu") and verbose:
        cmd.append("-Xptxas=-v")
    if src.endswith(".cpp"):
        cmd = [nvcc(), "-x", "c++"] + COMMON + ["-c", path, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"compiling {src} failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def build(force=False, verbose=False):
    """Compiles every translation unit and links the shared library; returns its path."""
    os.makedirs(BUILD, exist_ok=True)
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(lambda s: _compile(s, force, verbose), SOURCES))
    objs = [o for o, _ in results]
    if verbose:
        for (_, log), src in zip(results, SOURCES):
            if log:
                print(f"--- {src}\n{log}", file=sys.stderr)
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        cmd = [nvcc(), "-shared"] + ARCH + ["-Xcompiler", "-fPIC", "-o", LIB] + objs + LINK_LIBS
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"linking failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register / spill reports")
    a = ap.parse_args()
    print(build(a.force, a.verbose))
