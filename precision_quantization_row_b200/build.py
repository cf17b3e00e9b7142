"""Build step of libnvfp4pt.so (the CUDA library behind include/nvfp4pt.h).

nvcc compiles the kernels for sm_100a only; the library is written into this
package directory so that it travels with the source tree.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libnvfp4pt.so")
SOURCES = [os.path.join(CSRC, f) for f in ("nvfp4pt_api.cu", "nvfp4pt_noalloc.cu", "nvfp4pt_gemm.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("nvfp4pt_device.cuh", "nvfp4pt_kernels.cuh",
                                                  "nvfp4pt_rowpass.cuh", "nvfp4pt_colpass.cuh",
                                                  "nvfp4pt_dequant.cuh", "nvfp4pt_internal.h",
                                                  "nvfp4pt_gemm.cuh", "nvfp4pt_xform.cuh",
                                                  "nvfp4pt_requant.cuh", "nvfp4pt_colpass_tma.cuh",
                                                  "nvfp4pt_w2d.cuh")] + \
    [os.path.join(INCLUDE, f) for f in ("nvfp4pt.h", "nvfp4pt_timing.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

# Exactly one IEEE binary32 operation per step: no contraction into FMAs, IEEE
# division, no flush-to-zero. sm_100a only.
FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-fmad=false", "-prec-div=true", "-ftz=false",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, "-I", INCLUDE, "-I", CSRC, *SOURCES, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
