"""Test-only diagnostic library: the cast's device conversions over whole input domains.

libnvfp4pt_probe.so is built from nvfp4pt_probe.cu here, apart from the product library
libnvfp4pt.so, which exports only the cast's C ABI. It compiles the same device
functions (the package's csrc/nvfp4pt_device.cuh) that the cast kernels use.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
CSRC = os.path.join(ROOT, "precision_quantization_row_b200", "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libnvfp4pt_probe.so")
SOURCE = os.path.join(HERE, "nvfp4pt_probe.cu")
DEPS = [SOURCE, os.path.join(HERE, "nvfp4pt_probe.h"), os.path.join(CSRC, "nvfp4pt_device.cuh"),
        os.path.join(INCLUDE, "nvfp4pt.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
# The product library's flags (one IEEE operation per step, sm_100a only).
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-gencode", "arch=compute_100a,code=sm_100a",
         "-fmad=false", "-prec-div=true", "-ftz=false", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-fvisibility=hidden", "-shared", "-cudart", "static"]

EXPORTS = ("nvfp4pt_probe_transitions", "nvfp4pt_probe_pairs", "nvfp4pt_probe_e4m3_decode", "nvfp4pt_probe_div6",
           "nvfp4pt_probe_e4m3_div", "nvfp4pt_probe_pair_scales")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and all(os.path.getmtime(d) <= os.path.getmtime(LIB) for d in DEPS):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([NVCC, *FLAGS, "-I", HERE, "-I", INCLUDE, "-I", CSRC, SOURCE, "-o", tmp], check=True)
    os.replace(tmp, LIB)
    return LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.nvfp4pt_probe_transitions.argtypes = [I, P, ctypes.c_uint32, P, P]
        L.nvfp4pt_probe_pairs.argtypes = [P, I64, P, P]
        L.nvfp4pt_probe_e4m3_decode.argtypes = [P, P]
        L.nvfp4pt_probe_div6.argtypes = [P, P]
        L.nvfp4pt_probe_e4m3_div.argtypes = [I, I, P, P]
        L.nvfp4pt_probe_pair_scales.argtypes = [I, I, ctypes.c_uint32, P, P]
        for name in EXPORTS:
            getattr(L, name).restype = I
        _lib = L
    return _lib
