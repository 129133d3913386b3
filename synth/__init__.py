"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

The only code both sides use.  It draws iid N(0, 1) values and rounds them to
bf16 (bit patterns as numpy uint16); the generator is defined in ``gen.c``.
It holds none of the attention arithmetic.

Tensor streams: Q, K and V of one workload use tensor ids 0, 1 and 2 under the
same seed.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libsynth.so")

TENSOR_Q, TENSOR_K, TENSOR_V = 0, 1, 2


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _get():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.synth_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_void_p]
        L.synth_normal_bf16.restype = None
        _lib = L
    return _lib


def normal_bf16(shape, seed: int, tensor_id: int, out: np.ndarray | None = None) -> np.ndarray:
    """iid N(0, 1) rounded to bf16, as uint16 bit patterns of the given shape.

    ``out`` may be a preallocated contiguous uint16 array (e.g. a view of pinned
    host memory) of that many elements.
    """
    n = int(np.prod(shape, dtype=np.int64))
    if out is None:
        out = np.empty(shape, dtype=np.uint16)
    if out.dtype != np.uint16 or not out.flags.c_contiguous or out.size != n:
        raise ValueError("out must be a contiguous uint16 array of the right size")
    if n:
        _get().synth_normal_bf16(seed, tensor_id, 0, n, out.ctypes.data)
    return out.reshape(shape)


def bf16_bits_to_float(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (a.astype(np.uint32) << 16).view(np.float32)


def qkv(B: int, Hq: int, Hkv: int, N: int, D: int, seed: int = 0):
    """Q [B, Hq, N, D], K and V [B, Hkv, N, D] as bf16 bit patterns."""
    q = normal_bf16((B, Hq, N, D), seed, TENSOR_Q)
    k = normal_bf16((B, Hkv, N, D), seed, TENSOR_K)
    v = normal_bf16((B, Hkv, N, D), seed, TENSOR_V)
    return q, k, v
