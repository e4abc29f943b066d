"""Builds libpa.so (CUDA kernels + C ABI + host block manager) in-tree for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libpa.so")

CUDA_SOURCES = ["api.cu", "append.cu", "decode_simt.cu", "decode_tensor.cu", "decode_stream.cu", "merge.cu", "decode_noalloc.cu", "rope.cu", "prefill.cu", "prefill_tc.cu", "prefill_ws.cu"]
CXX_SOURCES = ["block_manager.cpp", "block_pool.cpp"]
HEADERS = ["pa_internal.h", "pa_device.cuh", "pa_ptx.cuh", "pa_umma.cuh"]

NVCC_FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-Xptxas", "-v"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    common = [os.path.join(INCLUDE, "pa.h")] + [os.path.join(CSRC, h) for h in HEADERS]
    objs = []
    for src in CUDA_SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        objs.append(o)
        if force or _stale(o, [s] + common):
            cmd = [_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", s, "-o", o]
            res = subprocess.run(cmd, capture_output=True, text=True)
            if res.returncode != 0:
                sys.stderr.write(res.stdout + res.stderr)
                raise RuntimeError("nvcc failed on %s" % src)
            with open(o + ".ptxas.txt", "w") as f:
                f.write(res.stderr)
            if verbose:
                sys.stderr.write(res.stderr)
    for src in CXX_SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        objs.append(o)
        if force or _stale(o, [s] + common):
            subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-fvisibility=hidden",
                                   "-I", INCLUDE, "-I", CSRC, "-c", s, "-o", o])
    if force or _stale(LIB, objs):
        tmp = LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call([_nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                               *objs, "-o", tmp, "-cudart", "static"])
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
