"""Builds and loads libcuda_conversions.so, the test-only wrapper around
CUDA's FP8 E4M3 / FP4 E2M1 conversions (cuda_conversions.cu beside this
file), used to pin the oracle's codebooks and rounding rule."""
from __future__ import annotations

import ctypes
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cuda_conversions.cu")
LIB = os.path.join(HERE, "libcuda_conversions.so")

_lib = None


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp"
    subprocess.run([os.environ.get("NVCC", "nvcc"), "-gencode", "arch=compute_100a,code=sm_100a", "-O2",
                    "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-o", tmp, SRC], check=True)
    os.replace(tmp, LIB)
    return LIB


def load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        f32p, u8p, vp = ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_uint8), ctypes.c_void_p
        for name in ("cvt_host_decode_e4m3", "cvt_host_decode_e2m1"):
            getattr(lib, name).argtypes = [f32p]
        for name in ("cvt_host_round_e4m3", "cvt_host_round_e2m1"):
            getattr(lib, name).argtypes = [f32p, u8p, ctypes.c_int]
        for name in ("cvt_dev_decode_e4m3", "cvt_dev_decode_e2m1"):
            getattr(lib, name).argtypes = [vp, vp]
        for name in ("cvt_dev_round_e4m3", "cvt_dev_round_e2m1"):
            getattr(lib, name).argtypes = [vp, vp, ctypes.c_int, vp]
        lib.cvt_host_e8m0_ceil.argtypes = [ctypes.POINTER(ctypes.c_double), u8p, ctypes.c_int]
        lib.cvt_host_decode_e8m0.argtypes = [f32p]
        lib.cvt_host_f32_to_bf16.argtypes = [f32p, ctypes.POINTER(ctypes.c_uint16), ctypes.c_int]
        _lib = lib
    return _lib
