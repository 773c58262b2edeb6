"""Build libmnb.so (the CUDA kernels + C ABI) in-tree for sm_100a with nvcc.

    python -m int4_block_quantized_matmulnbits_b200.build [-v] [--debug]

--debug links libmnb_debug.so instead: the same library with device-side
index checks in the kernels listed in DEBUG_SOURCES.

Each .cu file compiles to an object under _build/, then one shared library is
linked next to this file.  CUDA runtime is linked statically, so the library
only needs the NVIDIA driver at run time.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libmnb.so")
BUILD = os.path.join(ROOT, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills", "-I", os.path.join(ROOT, "include")]
SOURCES = ["api.cu", "quantize.cu", "gemv.cu", "gemv_tc.cu", "gemv_resident.cu", "gemv_chain.cu", "gemm_tcgen05.cu", "embed.cu", "gptq.cu"]
HEADERS = ["common.cuh", "internal.h"]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


# The debug build (libmnb_debug.so) compiles these files with device-side index
# checks (MNB_DEVICE_CHECKS); every other object is the release one.
DEBUG_SOURCES = ["gemv_resident.cu"]
DEBUG_OUT = os.path.join(HERE, "libmnb_debug.so")


def build(verbose: bool = False, ptxas_verbose: bool = False, debug: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", f) for f in ("mnb.h", "mnb_tune.h")]
    objs = []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        dbg = debug and src in DEBUG_SOURCES
        o = os.path.join(BUILD, src.replace(".cu", "_debug.o" if dbg else ".o"))
        objs.append(o)
        if _stale(o, [s] + hdrs) or ptxas_verbose:
            cmd = [NVCC, *ARCH, *FLAGS, *(["-DMNB_DEVICE_CHECKS=1"] if dbg else []), "-c", s, "-o", o]
            if ptxas_verbose:
                cmd += ["-Xptxas", "-v"]
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.check_call(cmd)
    out = DEBUG_OUT if debug else OUT
    if _stale(out, objs):
        tmp = out + ".tmp"
        cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, ptxas_verbose="--ptxas" in sys.argv, debug="--debug" in sys.argv))
