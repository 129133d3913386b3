"""CPU oracle for block-sparse causal attention, forward and backward (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never touches it, and the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP); this module only
builds it with gcc and marshals numpy arrays.  What each function computes, and
the passage of the pages it follows, is stated in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


class OraclePattern(ctypes.Structure):
    _fields_ = [
        ("causal", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("sinks", ctypes.c_int32),
        ("stride", ctypes.c_int32),
        ("n_global", ctypes.c_int32),
        ("global_rows_see_all", ctypes.c_int32),
        ("area", ctypes.c_int32),
        ("summary", ctypes.c_int32),
    ]


@dataclass(frozen=True)
class Pattern:
    """A fixed sparsity pattern: band of width ``window`` (inclusive, -1 for
    none; two-sided without causality), ``sinks`` leading key tokens, every
    ``stride``-th prior token (0 for none), ``n_global`` global tokens and, if
    ``area`` > 0, the pairs inside one stripe of ``area`` tokens, plus (``summary``
    > 0) keys in the last ``summary`` positions of any stripe."""

    window: int = -1
    sinks: int = 0
    stride: int = 0
    n_global: int = 0
    causal: int = 1
    global_rows_see_all: int = 0
    area: int = 0
    summary: int = 0

    def c(self) -> OraclePattern:
        return OraclePattern(self.causal, self.window, self.sinks, self.stride,
                             self.n_global, self.global_rows_see_all, self.area, self.summary)


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Oracle:
    """The compiled oracle at ``path`` (the default build, or a test's mutant)."""

    def __init__(self, path: str):
        L = ctypes.CDLL(path)
        P = ctypes.POINTER(OraclePattern)
        L.oracle_allowed.argtypes = [P, ctypes.c_int64, ctypes.c_int64]
        L.oracle_allowed.restype = ctypes.c_int
        L.oracle_count_pairs.argtypes = [P, ctypes.c_int64]
        L.oracle_count_pairs.restype = ctypes.c_int64
        L.oracle_row_counts.argtypes = [P, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        L.oracle_row_counts.restype = ctypes.c_int
        L.oracle_block_mask.argtypes = [P, ctypes.c_int64, ctypes.c_int32,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_block_mask.restype = ctypes.c_int64
        L.oracle_attention.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_int64, ctypes.c_int64, P, ctypes.c_double,
                                       ctypes.c_void_p, ctypes.c_int64,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32]
        L.oracle_attention.restype = ctypes.c_int
        d = ctypes.c_void_p
        L.oracle_attention_bwd.argtypes = [d, d, d, d, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_int64, ctypes.c_int64, P, ctypes.c_double,
                                           d, d, d, d, d, ctypes.c_int32]
        L.oracle_attention_bwd.restype = ctypes.c_int
        L.oracle_max_threads.argtypes = []
        L.oracle_max_threads.restype = ctypes.c_int
        self.L = L

    def allowed(self, p: Pattern, q: int, kv: int) -> bool:
        r = self.L.oracle_allowed(ctypes.byref(p.c()), q, kv)
        if r < 0:
            raise ValueError("pattern not defined by the oracle")
        return bool(r)

    def count_pairs(self, p: Pattern, N: int) -> int:
        return int(self.L.oracle_count_pairs(ctypes.byref(p.c()), N))

    def row_counts(self, p: Pattern, N: int, rows) -> np.ndarray:
        """Allowed keys of each of the given query rows (brute force per row)."""
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        out = np.zeros(len(rows), dtype=np.int64)
        if len(rows) and self.L.oracle_row_counts(ctypes.byref(p.c()), N, rows.ctypes.data, len(rows),
                                                  out.ctypes.data) != 0:
            raise ValueError("row outside [0, N)")
        return out

    def block_mask(self, p: Pattern, N: int, block: int):
        """Brute-force tile classification -> (counts[T], index[T, T], full[T, T])."""
        T = (N + block - 1) // block
        counts = np.zeros(T, dtype=np.int32)
        index = np.zeros((T, T), dtype=np.int32)
        full = np.zeros((T, T), dtype=np.uint8)
        live = self.L.oracle_block_mask(ctypes.byref(p.c()), N, block, counts.ctypes.data,
                                        index.ctypes.data, full.ctypes.data)
        if live < 0:
            raise ValueError("bad block-mask arguments")
        return counts, index, full

    def attention(self, q: np.ndarray, k: np.ndarray, v: np.ndarray, p: Pattern, scale: float,
                  rows: np.ndarray | None = None, n_threads: int = 0):
        """fp64 attention by definition.

        q: uint16 bf16 bits [B, Hq, N, D]; k, v: [B, Hkv, N, D].
        rows: optional int64 query positions.  Returns (O [B, Hq, R, D] float64,
        LSE [B, Hq, R] float64) with R = len(rows) or N.
        """
        for t in (q, k, v):
            if t.dtype != np.uint16 or not t.flags.c_contiguous:
                raise TypeError("inputs must be contiguous uint16 (bf16 bit patterns)")
        B, Hq, N, D = q.shape
        Hkv = k.shape[1]
        if k.shape != (B, Hkv, N, D) or v.shape != k.shape:
            raise ValueError("shape mismatch")
        if rows is None:
            R = N
            rows_ptr = None
        else:
            rows = np.ascontiguousarray(rows, dtype=np.int64)
            R = rows.shape[0]
            if R and (rows.min() < 0 or rows.max() >= N):
                raise ValueError("row out of range")
            rows_ptr = rows.ctypes.data
        O = np.empty((B, Hq, R, D), dtype=np.float64)
        LSE = np.empty((B, Hq, R), dtype=np.float64)
        rc = self.L.oracle_attention(q.ctypes.data, k.ctypes.data, v.ctypes.data, B, Hq, Hkv, N, D,
                                     ctypes.byref(p.c()), float(scale), rows_ptr, R,
                                     O.ctypes.data, LSE.ctypes.data, int(n_threads))
        if rc != 0:
            raise ValueError("bad attention arguments")
        return O, LSE

    def attention_bwd(self, q: np.ndarray, k: np.ndarray, v: np.ndarray, do: np.ndarray, p: Pattern,
                      scale: float, n_threads: int = 0):
        """fp64 gradients by definition.

        q, do: [B, Hq, N, D]; k, v: [B, Hkv, N, D]; either uint16 bf16 bit
        patterns (widened exactly) or float64.  Returns (O, LSE, dQ, dK, dV),
        float64, shapes as the inputs (LSE [B, Hq, N]).
        """
        def wide(a):
            if a.dtype == np.uint16:
                return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            if a.dtype != np.float64:
                raise TypeError("inputs must be uint16 (bf16 bit patterns) or float64")
            return np.ascontiguousarray(a)
        q, k, v, do = (wide(np.ascontiguousarray(a)) for a in (q, k, v, do))
        B, Hq, N, D = q.shape
        Hkv = k.shape[1]
        if k.shape != (B, Hkv, N, D) or v.shape != k.shape or do.shape != q.shape:
            raise ValueError("shape mismatch")
        O = np.empty_like(q)
        LSE = np.empty((B, Hq, N), dtype=np.float64)
        dQ, dK, dV = np.empty_like(q), np.empty_like(k), np.empty_like(v)
        rc = self.L.oracle_attention_bwd(q.ctypes.data, k.ctypes.data, v.ctypes.data, do.ctypes.data,
                                         B, Hq, Hkv, N, D, ctypes.byref(p.c()), float(scale),
                                         O.ctypes.data, LSE.ctypes.data, dQ.ctypes.data, dK.ctypes.data,
                                         dV.ctypes.data, int(n_threads))
        if rc != 0:
            raise ValueError("bad attention_bwd arguments")
        return O, LSE, dQ, dK, dV

    def max_threads(self) -> int:
        return int(self.L.oracle_max_threads())


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def allowed(p: Pattern, q: int, kv: int) -> bool:
    return default().allowed(p, q, kv)


def count_pairs(p: Pattern, N: int) -> int:
    return default().count_pairs(p, N)


def row_counts(p: Pattern, N: int, rows) -> np.ndarray:
    return default().row_counts(p, N, rows)


def block_mask(p: Pattern, N: int, block: int):
    return default().block_mask(p, N, block)


def attention(q, k, v, p: Pattern, scale: float, rows=None, n_threads: int = 0):
    return default().attention(q, k, v, p, scale, rows=rows, n_threads=n_threads)


def attention_bwd(q, k, v, do, p: Pattern, scale: float, n_threads: int = 0):
    return default().attention_bwd(q, k, v, do, p, scale, n_threads=n_threads)


def max_threads() -> int:
    return default().max_threads()


def compile_source(src_text: str, out_path: str) -> str:
    """Compile oracle source text (a test's mutant of oracle.c) to ``out_path``."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           "-o", out_path, c_path, "-lm"])
    return out_path


def source() -> str:
    with open(_SRC) as f:
        return f.read()
