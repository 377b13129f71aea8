"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the CPU oracle.

Holds none of the attention method's arithmetic: only a counter-based normal
generator (SplitMix64 + Box-Muller, see synth.c) and the table of workload
shapes.  Floating-point tensors come back as numpy arrays: float32 for fp32
storage, uint16 bit patterns for bfloat16 storage.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None

KIND_F64, KIND_F32, KIND_BF16 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so (gcc, OpenMP) if missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                                     ctypes.c_double, ctypes.c_int, ctypes.c_void_p]
        lib.synth_normal.restype = None
        lib.synth_splitmix64_nth.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_splitmix64_nth.restype = ctypes.c_uint64
        lib.synth_round_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        lib.synth_round_bf16.restype = None
        _lib = lib
    return _lib


def splitmix64_nth(state: int, n: int) -> int:
    return int(_load().synth_splitmix64_nth(state, n))


def round_bf16_bits(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().synth_round_bf16(x.ctypes.data, x.size, out.ctypes.data)
    return out


def normal(seed: int, tensor_id: int, shape, std: float, kind: int, offset: int = 0, out=None) -> np.ndarray:
    """N(0, std^2) samples for elements [offset, offset + prod(shape)) of tensor `tensor_id`."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    dt = {KIND_F64: np.float64, KIND_F32: np.float32, KIND_BF16: np.uint16}[kind]
    if out is None:
        out = np.empty(shape, dtype=dt)
    assert out.dtype == dt and out.flags.c_contiguous and out.size == n
    if n:
        _load().synth_normal(seed, tensor_id, offset, n, float(std), kind, out.ctypes.data)
    return out


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32)


from .workloads import *  # noqa: E402,F401,F403
