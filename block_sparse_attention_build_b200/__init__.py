"""Block-sparse causal attention forward and backward on B200 (sm_100a).

Thin binding over the C ABI in ``include/sparse_attn.h`` (``libsparse_attn.so``,
built in-tree).  This module only marshals arguments: torch tensors supply
device memory and the CUDA stream; every step of the computation runs in the
library's CUDA kernel.  There is no CPU fallback: if the library is missing or
fails to load, importing this package raises.

    mask = build_block_mask(Pattern(window=1024, sinks=4), N=8192, block=128)
    dmask = mask.to_device("cuda")
    O, LSE = fwd(Q, K, V, dmask, Pattern(window=1024, sinks=4))
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsparse_attn.so")

SA_OK = 0
SA_ERR_INVALID_ARG = -1
SA_ERR_UNSUPPORTED = -2
SA_ERR_MISALIGNED = -3
SA_ERR_BUFFER_TOO_SMALL = -4
SA_ERR_CUDA = -5
SA_ERR_DEVICE_TIMEOUT = -6
SA_ERR_MASK_MISMATCH = -7
SA_ERR_SCRATCH_TOO_SMALL = -8
NOALLOC_SCRATCH_BYTES = 1 << 20

DEBUG_SKIP_Q_LOAD = 1
DEBUG_SPLIT_ALL = 2
DEBUG_BWD_SPLIT = 4

EXPORTED = (
    "sparse_attn_num_tiles", "sparse_attn_build_block_mask", "sparse_attn_count_pairs",
    "sparse_attn_fwd", "sparse_attn_fwd_host", "sparse_attn_fwd_host_async", "sparse_attn_fwd_host_workspace",
    "sparse_attn_check_device", "sparse_attn_set_debug", "sparse_attn_status_string",
    "sparse_attn_version", "sparse_attn_fwd_noalloc", "sparse_attn_fwd_heads",
    "sparse_attn_transpose_block_mask", "sparse_attn_bwd_workspace", "sparse_attn_bwd",
    "sparse_attn_stride_plan", "sparse_attn_fwd_stride_workspace", "sparse_attn_fwd_stride",
    "sparse_attn_bwd_heads",
)


class SparseAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class _Pattern(ctypes.Structure):
    _fields_ = [("causal", ctypes.c_int32), ("window", ctypes.c_int32), ("sinks", ctypes.c_int32),
                ("stride", ctypes.c_int32), ("n_global", ctypes.c_int32), ("area", ctypes.c_int32),
                ("summary", ctypes.c_int32)]


class _BlockMask(ctypes.Structure):
    _fields_ = [("n_q_tiles", ctypes.c_int32), ("n_kv_tiles", ctypes.c_int32), ("block", ctypes.c_int32),
                ("max_per_row", ctypes.c_int32), ("n_live", ctypes.c_int64), ("n_full", ctypes.c_int64),
                ("kv_count", ctypes.c_void_p), ("kv_index", ctypes.c_void_p), ("kv_full", ctypes.c_void_p)]


class _Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("N", ctypes.c_int32), ("D", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          f"`python -m block_sparse_attention_build_b200._build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    P, M, S = ctypes.POINTER(_Pattern), ctypes.POINTER(_BlockMask), ctypes.POINTER(_Shape)
    vp = ctypes.c_void_p
    L.sparse_attn_num_tiles.argtypes = [ctypes.c_int64, ctypes.c_int32]
    L.sparse_attn_num_tiles.restype = ctypes.c_int32
    L.sparse_attn_build_block_mask.argtypes = [P, ctypes.c_int64, ctypes.c_int32, M]
    L.sparse_attn_count_pairs.argtypes = [P, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)]
    L.sparse_attn_fwd.argtypes = [vp, vp, vp, M, P, S, ctypes.c_float, vp, vp, vp]
    L.sparse_attn_fwd_host.argtypes = [vp, vp, vp, M, P, S, ctypes.c_float, vp, vp, vp, ctypes.c_size_t, vp]
    L.sparse_attn_fwd_host_async.argtypes = [vp, vp, vp, M, P, S, ctypes.c_float, vp, vp, vp, ctypes.c_size_t, vp]
    L.sparse_attn_fwd_host_workspace.argtypes = [S, ctypes.POINTER(ctypes.c_size_t)]
    L.sparse_attn_fwd_noalloc.argtypes = [vp, vp, vp, M, P, S, ctypes.c_float, vp, vp, vp]
    L.sparse_attn_fwd_heads.argtypes = [vp, vp, vp, M, P, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32), S,
                                        ctypes.c_float, vp, vp, vp]
    L.sparse_attn_transpose_block_mask.argtypes = [M, M]
    L.sparse_attn_bwd_workspace.argtypes = [S, ctypes.POINTER(ctypes.c_size_t)]
    L.sparse_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, M, P, S, ctypes.c_float, vp, vp, vp, vp,
                                  ctypes.c_size_t, vp]
    L.sparse_attn_stride_plan.argtypes = [P, ctypes.c_int64, ctypes.c_int32, M, M]
    L.sparse_attn_fwd_stride_workspace.argtypes = [S, ctypes.POINTER(ctypes.c_size_t)]
    L.sparse_attn_fwd_stride.argtypes = [vp, vp, vp, M, M, P, S, ctypes.c_float, vp, vp, vp, ctypes.c_size_t, vp]
    L.sparse_attn_bwd_heads.argtypes = [vp, vp, vp, vp, vp, vp, M, P, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32),
                                        S, ctypes.c_float, vp, vp, vp, vp, ctypes.c_size_t, vp]
    L.sparse_attn_check_device.argtypes = [vp]
    L.sparse_attn_set_debug.argtypes = [ctypes.c_int32, ctypes.c_int64]
    L.sparse_attn_status_string.argtypes = [ctypes.c_int]
    L.sparse_attn_status_string.restype = ctypes.c_char_p
    L.sparse_attn_version.argtypes = []
    L.sparse_attn_version.restype = ctypes.c_int32
    for name in ("sparse_attn_build_block_mask", "sparse_attn_count_pairs", "sparse_attn_fwd",
                 "sparse_attn_fwd_host", "sparse_attn_fwd_host_async", "sparse_attn_fwd_host_workspace",
                 "sparse_attn_check_device",
                 "sparse_attn_set_debug", "sparse_attn_fwd_noalloc", "sparse_attn_fwd_heads",
                 "sparse_attn_transpose_block_mask", "sparse_attn_bwd_workspace", "sparse_attn_bwd",
                 "sparse_attn_stride_plan", "sparse_attn_fwd_stride_workspace", "sparse_attn_fwd_stride",
                 "sparse_attn_bwd_heads"):
        getattr(L, name).restype = ctypes.c_int
    return L


lib = _load()


def status_string(status: int) -> str:
    return lib.sparse_attn_status_string(status).decode()


def _check(status: int, where: str) -> None:
    if status != SA_OK:
        raise SparseAttnError(status, where)


@dataclass(frozen=True)
class Pattern:
    """allowed(q, kv) = (not causal or q >= kv) and ((window >= 0 and |q - kv| <= window)
    or kv < sinks or (stride > 0 and (q - kv) % stride == 0) or kv < n_global or q < n_global
    or (area > 0 and q // area == kv // area)
    or (area > 0 and summary > 0 and kv % area >= area - summary)).  A stride needs causal = 1."""

    window: int = -1
    sinks: int = 0
    stride: int = 0
    n_global: int = 0
    causal: int = 1
    area: int = 0
    summary: int = 0

    def _c(self) -> _Pattern:
        return _Pattern(self.causal, self.window, self.sinks, self.stride, self.n_global, self.area, self.summary)


class BlockMask:
    """Per-query-tile lists of live kv tiles and their full flags (host numpy
    arrays, or torch tensors on a device after ``to_device``)."""

    def __init__(self, counts, index, full, block: int, n_live: int, n_full: int, max_per_row: int, N: int):
        self.counts, self.index, self.full = counts, index, full
        self.block, self.n_live, self.n_full, self.max_per_row, self.N = block, n_live, n_full, max_per_row, N

    @property
    def T(self) -> int:
        return int(self.counts.shape[0])

    def _ptr(self, a) -> int:
        return a.data_ptr() if hasattr(a, "data_ptr") else a.ctypes.data

    def _c(self) -> _BlockMask:
        T = self.T
        return _BlockMask(T, T, self.block, self.max_per_row, self.n_live, self.n_full,
                          self._ptr(self.counts) if T else None, self._ptr(self.index) if T else None,
                          self._ptr(self.full) if T else None)

    @property
    def on_host(self) -> bool:
        return isinstance(self.counts, np.ndarray)

    def to_device(self, device) -> "BlockMask":
        import torch
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        return BlockMask(t(self.counts), t(self.index), t(self.full), self.block, self.n_live,
                         self.n_full, self.max_per_row, self.N)


def _host_masks(where: str, *masks) -> None:
    """The call reads the mask's arrays on the host: numpy, not a device copy
    (whose addresses the host cannot read)."""
    for m in masks:
        if not m.on_host:
            raise TypeError(f"{where} takes the host block mask (numpy arrays), not a device copy")


def _device_masks(where: str, device, *masks) -> None:
    """The call's kernels read the mask's arrays: a copy on the tensors' device
    (``to_device``), not host arrays."""
    for m in masks:
        c = m.counts
        if m.on_host or not getattr(c, "is_cuda", False) or c.device != device:
            raise TypeError(f"{where} takes the block mask on the tensors' device (BlockMask.to_device)")


def num_tiles(N: int, block: int) -> int:
    T = lib.sparse_attn_num_tiles(N, block)
    if T < 0:
        raise SparseAttnError(T, "sparse_attn_num_tiles")
    return T


def build_block_mask(pattern: Pattern, N: int, block: int = 128) -> BlockMask:
    """Compile ``pattern`` over an N x N causal score matrix into block x block tiles."""
    T = max(num_tiles(N, block), 0)
    counts = np.zeros(T, dtype=np.int32)
    index = np.zeros((T, T), dtype=np.int32)
    full = np.zeros((T, T), dtype=np.uint8)
    m = _BlockMask(T, T, 0, 0, 0, 0, counts.ctypes.data if T else None,
                   index.ctypes.data if T else None, full.ctypes.data if T else None)
    _check(lib.sparse_attn_build_block_mask(ctypes.byref(pattern._c()), N, block, ctypes.byref(m)),
           "sparse_attn_build_block_mask")
    return BlockMask(counts, index, full, m.block, m.n_live, m.n_full, m.max_per_row, N)


def transpose_block_mask(mask: BlockMask) -> BlockMask:
    """Per-kv-tile lists of the query tiles that attend to it (host arrays);
    ``counts[c]``, ``index[c, e]`` and ``full[c, e]`` with rows and columns
    swapped relative to ``mask``.  The backward pass takes this form."""
    _host_masks("transpose_block_mask", mask)
    T = mask.T
    counts = np.zeros(T, dtype=np.int32)
    index = np.zeros((T, T), dtype=np.int32)
    full = np.zeros((T, T), dtype=np.uint8)
    out = _BlockMask(T, T, 0, 0, 0, 0, counts.ctypes.data if T else None,
                     index.ctypes.data if T else None, full.ctypes.data if T else None)
    src = mask._c()
    _check(lib.sparse_attn_transpose_block_mask(ctypes.byref(src), ctypes.byref(out)),
           "sparse_attn_transpose_block_mask")
    return BlockMask(counts, index, full, out.block, out.n_live, out.n_full, out.max_per_row, mask.N)


def stride_plan(pattern: Pattern, N: int, block: int = 128):
    """(pass1, pass2) host block masks of the stride-aware path (see
    ``fwd_stride``): the pattern without its stride in token order, and the
    remaining stride pairs on tokens grouped by residue."""
    T = max(num_tiles(N, block), 0)
    arrays = []
    cms = []
    for _ in range(2):
        a = (np.zeros(T, dtype=np.int32), np.zeros((T, T), dtype=np.int32), np.zeros((T, T), dtype=np.uint8))
        arrays.append(a)
        cms.append(_BlockMask(T, T, 0, 0, 0, 0, a[0].ctypes.data if T else None, a[1].ctypes.data if T else None,
                              a[2].ctypes.data if T else None))
    _check(lib.sparse_attn_stride_plan(ctypes.byref(pattern._c()), N, block, ctypes.byref(cms[0]),
                                       ctypes.byref(cms[1])), "sparse_attn_stride_plan")
    return tuple(BlockMask(a[0], a[1], a[2], m.block, m.n_live, m.n_full, m.max_per_row, N)
                 for a, m in zip(arrays, cms))


def count_pairs(pattern: Pattern, N: int) -> int:
    out = ctypes.c_int64(0)
    _check(lib.sparse_attn_count_pairs(ctypes.byref(pattern._c()), N, ctypes.byref(out)),
           "sparse_attn_count_pairs")
    return out.value


def _stream_handle(stream, device) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def fwd(q, k, v, mask: BlockMask, pattern: Pattern, scale: float | None = None, out=None, lse=None,
        stream=None):
    """O [B, Hq, N, D] bf16 and LSE [B, Hq, N] fp32 on q's device.

    q: [B, Hq, N, D] bf16 CUDA tensor; k, v: [B, Hkv, N, D].  ``mask`` must be
    on the same device.  Asynchronous on ``stream`` (default: current stream).
    """
    import torch
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise TypeError("q, k, v must be contiguous bf16 CUDA tensors")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _device_masks("fwd", q.device, mask)
    shape = _Shape(B, Hq, Hkv, N, D)
    with torch.cuda.device(q.device):
        st = _stream_handle(stream, q.device)
        _check(lib.sparse_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(mask._c()),
                                   ctypes.byref(pattern._c()), ctypes.byref(shape), float(scale),
                                   out.data_ptr(), lse.data_ptr(), st), "sparse_attn_fwd")
    return out, lse


def fwd_heads(q, k, v, masks, patterns, head_pattern, scale: float | None = None, out=None, lse=None,
              stream=None):
    """Forward pass with a pattern per query head: head h attends under
    ``patterns[head_pattern[h]]`` with the device block mask ``masks[head_pattern[h]]``.

    ``masks`` and ``patterns`` are sequences of equal length (1..8);
    ``head_pattern`` holds Hq ints.  Otherwise as ``fwd``.
    """
    import torch
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise TypeError("q, k, v must be contiguous bf16 CUDA tensors")
    if len(masks) != len(patterns):
        raise ValueError("one block mask per pattern")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    n = len(patterns)
    cmasks = (_BlockMask * max(n, 1))(*[m._c() for m in masks])
    cpats = (_Pattern * max(n, 1))(*[p_._c() for p_ in patterns])
    heads = (ctypes.c_int32 * max(len(head_pattern), 1))(*[int(h) for h in head_pattern])
    _device_masks("fwd_heads", q.device, *masks)
    shape = _Shape(B, Hq, Hkv, N, D)
    with torch.cuda.device(q.device):
        st = _stream_handle(stream, q.device)
        _check(lib.sparse_attn_fwd_heads(q.data_ptr(), k.data_ptr(), v.data_ptr(), cmasks, cpats, n, heads,
                                         ctypes.byref(shape), float(scale), out.data_ptr(), lse.data_ptr(), st),
               "sparse_attn_fwd_heads")
    return out, lse


def bwd_workspace_bytes(B: int, Hq: int, Hkv: int, N: int, D: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.sparse_attn_bwd_workspace(ctypes.byref(_Shape(B, Hq, Hkv, N, D)), ctypes.byref(n)),
           "sparse_attn_bwd_workspace")
    return n.value


def bwd(q, k, v, o, lse, do, mask_t: BlockMask, pattern: Pattern, scale: float | None = None,
        dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients (dQ, dK, dV) for the upstream gradient ``do``.

    q, o, do: [B, Hq, N, D] bf16 CUDA tensors; k, v: [B, Hkv, N, D]; lse: the
    forward's [B, Hq, N] fp32.  ``mask_t`` is ``transpose_block_mask`` of the
    pattern's block-128 mask, on the same device.  Asynchronous on ``stream``.
    """
    import torch
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    for t in (q, k, v, o, do):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise TypeError("q, k, v, o, do must be contiguous bf16 CUDA tensors")
    if lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous():
        raise TypeError("lse must be a contiguous fp32 CUDA tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = bwd_workspace_bytes(B, Hq, Hkv, N, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _device_masks("bwd", q.device, mask_t)
    shape = _Shape(B, Hq, Hkv, N, D)
    with torch.cuda.device(q.device):
        st = _stream_handle(stream, q.device)
        _check(lib.sparse_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                   do.data_ptr(), ctypes.byref(mask_t._c()), ctypes.byref(pattern._c()),
                                   ctypes.byref(shape), float(scale), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                   workspace.data_ptr(), workspace.numel(), st), "sparse_attn_bwd")
    return dq, dk, dv


def fwd_stride_workspace_bytes(B: int, Hq: int, Hkv: int, N: int, D: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.sparse_attn_fwd_stride_workspace(ctypes.byref(_Shape(B, Hq, Hkv, N, D)), ctypes.byref(n)),
           "sparse_attn_fwd_stride_workspace")
    return n.value


def fwd_stride(q, k, v, pass1: BlockMask, pass2: BlockMask, pattern: Pattern, scale: float | None = None,
               out=None, lse=None, workspace=None, stream=None):
    """Forward pass of a strided pattern by the stride-aware path (``stride_plan``'s
    masks on q's device); same results as ``fwd`` with the whole pattern."""
    import torch
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise TypeError("q, k, v must be contiguous bf16 CUDA tensors")
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _device_masks("fwd_stride", q.device, pass1, pass2)
    shape = _Shape(B, Hq, Hkv, N, D)
    n = ctypes.c_size_t(0)
    _check(lib.sparse_attn_fwd_stride_workspace(ctypes.byref(shape), ctypes.byref(n)), "sparse_attn_fwd_stride_workspace")
    if workspace is None:
        workspace = torch.empty(max(n.value, 1), dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        st = _stream_handle(stream, q.device)
        _check(lib.sparse_attn_fwd_stride(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(pass1._c()),
                                          ctypes.byref(pass2._c()), ctypes.byref(pattern._c()), ctypes.byref(shape),
                                          float(scale), out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                                          workspace.numel(), st), "sparse_attn_fwd_stride")
    return out, lse


def bwd_heads(q, k, v, o, lse, do, masks_t, patterns, head_pattern, scale: float | None = None,
              dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients with a pattern per query head: head h under ``patterns[head_pattern[h]]``
    with the transposed device mask ``masks_t[head_pattern[h]]``.  Otherwise as ``bwd``."""
    import torch
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    for t in (q, k, v, o, do):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise TypeError("q, k, v, o, do must be contiguous bf16 CUDA tensors")
    if len(masks_t) != len(patterns):
        raise ValueError("one transposed block mask per pattern")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = bwd_workspace_bytes(B, Hq, Hkv, N, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    n = len(patterns)
    cmasks = (_BlockMask * max(n, 1))(*[m._c() for m in masks_t])
    cpats = (_Pattern * max(n, 1))(*[p_._c() for p_ in patterns])
    heads = (ctypes.c_int32 * max(len(head_pattern), 1))(*[int(h) for h in head_pattern])
    _device_masks("bwd_heads", q.device, *masks_t)
    shape = _Shape(B, Hq, Hkv, N, D)
    with torch.cuda.device(q.device):
        st = _stream_handle(stream, q.device)
        _check(lib.sparse_attn_bwd_heads(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                         do.data_ptr(), cmasks, cpats, n, heads, ctypes.byref(shape), float(scale),
                                         dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                                         workspace.numel(), st), "sparse_attn_bwd_heads")
    return dq, dk, dv


def fwd_host_workspace_bytes(B: int, Hq: int, Hkv: int, N: int, D: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.sparse_attn_fwd_host_workspace(ctypes.byref(_Shape(B, Hq, Hkv, N, D)), ctypes.byref(n)),
           "sparse_attn_fwd_host_workspace")
    return n.value


def fwd_host(q_host, k_host, v_host, mask: BlockMask, pattern: Pattern, o_host, lse_host, workspace,
             scale: float | None = None, stream=None, wait: bool = True) -> None:
    """Forward from host (ideally pinned) tensors: copies in, computes, copies
    out and waits, in chunks of kv heads whose copies overlap the kernels.
    ``workspace`` is a device tensor of at least ``fwd_host_workspace_bytes``
    bytes; ``mask`` is the HOST block mask from ``build_block_mask``.  With
    ``wait=False`` the call only queues the work (sparse_attn_fwd_host_async):
    ``stream`` reaches its end once O and LSE are in host memory, and successive
    calls overlap their input and output copies."""
    _host_masks("fwd_host", mask)
    B, Hq, N, D = q_host.shape
    Hkv = k_host.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    shape = _Shape(B, Hq, Hkv, N, D)
    nbytes = workspace.numel() * workspace.element_size()
    import torch
    with torch.cuda.device(workspace.device):
        st = _stream_handle(stream, workspace.device)
        fn = lib.sparse_attn_fwd_host if wait else lib.sparse_attn_fwd_host_async
        _check(fn(q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(), ctypes.byref(mask._c()),
                  ctypes.byref(pattern._c()), ctypes.byref(shape), float(scale), o_host.data_ptr(),
                  lse_host.data_ptr(), workspace.data_ptr(), nbytes, st),
               "sparse_attn_fwd_host" if wait else "sparse_attn_fwd_host_async")


def fwd_noalloc(q, k, v, mask: BlockMask, pattern: Pattern, out, lse, scale: float | None = None,
                stream=None) -> None:
    """The forward pass for callers that cannot allocate device memory.

    ``mask`` is the HOST block mask from ``build_block_mask``; ``out`` and
    ``lse`` are caller-allocated device tensors.  The library keeps its scratch
    (status word, device copy of the mask) in a static device array of
    ``NOALLOC_SCRATCH_BYTES``; the call waits for the stream and raises on a
    device timeout or a mask too large for that array.
    """
    import torch
    B, Hq, N, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    _host_masks("fwd_noalloc", mask)
    shape = _Shape(B, Hq, k.shape[1], N, D)
    with torch.cuda.device(q.device):
        st = _stream_handle(stream, q.device)
        _check(lib.sparse_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(mask._c()),
                                           ctypes.byref(pattern._c()), ctypes.byref(shape), float(scale),
                                           out.data_ptr(), lse.data_ptr(), st), "sparse_attn_fwd_noalloc")


def check_device(stream=None, device=None) -> int:
    """Wait for the stream and return the kernel status (SA_OK or SA_ERR_DEVICE_TIMEOUT)."""
    import torch
    dev = device if device is not None else torch.cuda.current_device()
    with torch.cuda.device(dev):
        return lib.sparse_attn_check_device(_stream_handle(stream, dev))


def set_debug(flags: int = 0, timeout_cycles: int = 0) -> None:
    _check(lib.sparse_attn_set_debug(flags, timeout_cycles), "sparse_attn_set_debug")


def version() -> int:
    return int(lib.sparse_attn_version())
