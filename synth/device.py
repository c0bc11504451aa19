"""Fill device caches with the seeded generator's values, on the GPU.

Calls the device twin (``synth/csrc/synth_gen.cu``, built into
``synth/_lib/libsynth.so``), which reproduces ``synth.cache_rows`` bit for bit.
Only used to create large inputs quickly; it draws inputs and nothing else.
"""
import ctypes
import os
import subprocess

import numpy as np

from . import normal, workload

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libsynth.so")
_lib = None
MAX_D = 128


def build(verbose=False):
    os.makedirs(os.path.dirname(LIB_PATH), exist_ok=True)
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
           "-fmad=false", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
           "-o", LIB_PATH, os.path.join(_HERE, "csrc", "synth_gen.cu")]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return LIB_PATH


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise FileNotFoundError(f"{LIB_PATH} is not built; call synth.device.build()")
        lib = ctypes.CDLL(LIB_PATH)
        lib.synth_fill.restype = ctypes.c_int
        lib.synth_fill.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                   ctypes.c_int32, ctypes.c_int32, ctypes.c_uint32,
                                   ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32,
                                   ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32,
                                   ctypes.c_void_p, ctypes.c_void_p]
        _lib = lib
    return _lib


def _consts(w, layer):
    u = np.zeros(MAX_D)
    u[:w.d] = workload.unit_direction(w.seed, layer, w.d)
    c = (list(normal.ATANH_C) + list(normal.SIN_C) + list(normal.COS_C)
         + [normal.LN2, normal.HALF_PI, normal.SQRT2] + list(u)
         + [workload.PLANT_SCALE, workload.PLANT_NOISE])
    return np.ascontiguousarray(np.array(c, dtype=np.float64))


def fill(tensor, w, layer, kind, T=None, stream=0):
    """Fill a contiguous device tensor [B][H][cap][d] (torch, float32 or
    int16/uint16-as-bf16 bits) with cache ``kind`` of workload ``w``, tokens
    t < T (default: cap). Rows beyond T are left as they are."""
    import torch
    B, H, cap, d = tensor.shape
    assert tensor.is_contiguous() and d == w.d
    T = cap if T is None else T
    tid = {"K": workload.T_K, "V": workload.T_V, "KD": workload.T_KD, "VD": workload.T_VD}[kind]
    plant = kind in ("K", "KD")
    consts = _consts(w, layer)
    dt = 0 if w.dtype == workload.F32 else 1
    if isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    rc = _load().synth_fill(
        ctypes.c_void_p(tensor.data_ptr()), H * cap * d, cap * d, T, B, H, d, dt,
        w.seed & 0xFFFFFFFF, tid, layer, int(plant), workload.T_PLANT,
        0 if kind == "K" else 1000, workload.PLANT_THRESH,
        consts.ctypes.data_as(ctypes.c_void_p), ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"synth_fill failed with CUDA error {rc}")
