"""Seeded synthetic inputs shared by the CUDA path and the CPU oracle.

This package holds no arithmetic of the MoE layer.  It turns a seed, a tensor
id and an element index into a reproducible number (Philox4x32-10 plus
Box-Muller, see ``philox_normal.c``) and rounds it once to the storage type,
so both sides of every parity check read bit-identical inputs.  bf16 tensors
are returned as ``numpy.uint16`` arrays holding the raw bf16 bits.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "philox_normal.c")
_LIB = os.path.join(_HERE, "_synth.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the generator with gcc (OpenMP) next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, dbl, vp = ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p
            for name in ("synth_normal_f64", "synth_normal_f32", "synth_normal_bf16"):
                fn = getattr(lib, name)
                fn.argtypes = [u64, u64, u64, u64, dbl, dbl, vp]
                fn.restype = None
            lib.synth_philox4x32_10.argtypes = [vp, vp, vp]
            lib.synth_philox4x32_10.restype = None
            lib.synth_round_bf16.argtypes = [vp, u64, vp]
            lib.synth_round_bf16.restype = None
            _lib = lib
    return _lib


def philox4x32_10(ctr, key):
    """One Philox4x32-10 block: returns 4 uint32 words."""
    lib = _load()
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    lib.synth_philox4x32_10(c.ctypes.data, k.ctypes.data, out.ctypes.data)
    return out


def round_bf16(values) -> np.ndarray:
    """Round doubles to bf16 bits (nearest, ties to even)."""
    lib = _load()
    v = np.ascontiguousarray(values, dtype=np.float64).ravel()
    out = np.empty(v.size, dtype=np.uint16)
    lib.synth_round_bf16(v.ctypes.data, v.size, out.ctypes.data)
    return out


def normal(seed: int, tensor_id: int, shape, std: float = 1.0, mean: float = 0.0,
           dtype: str = "f64", start: int = 0) -> np.ndarray:
    """Elements [start, start + prod(shape)) of tensor ``tensor_id``.

    dtype: "f64" (unrounded), "f32", or "bf16" (uint16 bit patterns).
    """
    lib = _load()
    shape = tuple(int(s) for s in (shape if hasattr(shape, "__len__") else (shape,)))
    n = int(np.prod(shape)) if shape else 1
    if dtype == "f64":
        out = np.empty(n, dtype=np.float64)
        fn = lib.synth_normal_f64
    elif dtype == "f32":
        out = np.empty(n, dtype=np.float32)
        fn = lib.synth_normal_f32
    elif dtype == "bf16":
        out = np.empty(n, dtype=np.uint16)
        fn = lib.synth_normal_bf16
    else:
        raise ValueError(f"unknown dtype {dtype!r}")
    if n:
        fn(seed, tensor_id, start, n, float(mean), float(std), out.ctypes.data)
    return out.reshape(shape)
