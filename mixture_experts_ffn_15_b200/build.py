"""Build libmoe_b200.so in-tree with nvcc for sm_100a.

    python -m mixture_experts_ffn_15_b200.build [--force] [--ptxas-v]

Each CUDA source is compiled to an object under _build/ (in parallel), then the
objects are linked into mixture_experts_ffn_15_b200/libmoe_b200.so with the CUDA
runtime linked statically.  The driver API entry point for tensor-map encoding is
fetched at run time, so the library does not link libcuda.
"""
import argparse
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")
SOURCES = ["api.cu", "route.cu", "route_small.cu", "permute.cu", "combine.cu", "ffn_simt.cu",
           "gemm_tc.cu", "route_tc.cu", "gemm_pair.cu", "static_scratch.cu", "rmsnorm.cu"]
HEADERS = ["common.cuh", "sm100.cuh", "kernels.h", "combine.cuh", "topk_warp.cuh", "tile_map.cuh",
           "tmap.cuh", "tc_common.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc():
    exe = shutil.which("nvcc")
    if exe is None and os.path.exists("/usr/local/cuda/bin/nvcc"):
        exe = "/usr/local/cuda/bin/nvcc"
    if exe is None:
        raise RuntimeError("nvcc not found")
    return exe


def _compile(src, ptxas_v):
    obj = os.path.join(BUILD_DIR, os.path.splitext(src)[0] + ".o")
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC",
           "-I", INCLUDE, "-I", CSRC, "-c", os.path.join(CSRC, src), "-o", obj]
    if ptxas_v:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr}")
    return obj, r.stderr


def _stale():
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps += [os.path.join(INCLUDE, "moe_b200.h"), os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force=False, ptxas_v=False, verbose=False):
    """Compile every source for sm_100a and link the shared library."""
    if not force and not _stale():
        return LIB_PATH
    os.makedirs(BUILD_DIR, exist_ok=True)
    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(lambda s: _compile(s, ptxas_v), SOURCES))
    if verbose or ptxas_v:
        for (_, log) in results:
            if log:
                print(log, file=sys.stderr)
    objs = [o for (o, _) in results]
    tmp = LIB_PATH + ".tmp"
    cmd = [nvcc(), "-shared", *ARCH, "-Xcompiler", "-fPIC", "-cudart", "static", *objs, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_v=a.ptxas_v, verbose=True))
