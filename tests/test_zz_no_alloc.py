"""The no-allocation forward entry point, for callers that cannot allocate
device memory (a program that reserves all of it up front in its own pool and
must not call cudaMalloc on the request path).

It runs the same kernel as sparse_attn_fwd, with the kernel's scratch (status
word, device copy of the block mask) in a static device array of the library.
Checked here through the C ABI: two calls in a row, with different shapes and
patterns so the shared scratch is rewritten, each bit for bit against
sparse_attn_fwd on the same inputs and within the parity bars against the
oracle; and a device timeout reported through the static status word.  This
file is collected last so that a stop at the first failure has run everything
else.
"""
import ctypes
import math

import numpy as np
import pytest

import block_sparse_attention_build_b200 as sa
import synth

O_TOL = 2e-2
LSE_TOL = 1e-3


def test_mask_larger_than_scratch_is_rejected_before_device_work():
    # T = 458 tiles per side needs 256 + 4 T + 5 T^2 bytes (with alignment) > 1 MiB
    N, block = 458 * 128, 128
    mask = sa.build_block_mask(sa.Pattern(window=64), N, block)
    shape = sa._Shape(1, 1, 1, N, 128)
    fake = 1 << 20  # never dereferenced: the size check comes first
    rc = sa.lib.sparse_attn_fwd_noalloc(fake, fake, fake, ctypes.byref(mask._c()),
                                        ctypes.byref(sa.Pattern(window=64)._c()), ctypes.byref(shape), 0.1,
                                        fake, fake, None)
    assert rc == sa.SA_ERR_SCRATCH_TOO_SMALL
    assert "static scratch" in sa.status_string(rc)


def _noalloc(q, k, v, host_mask, p, scale, O, L):
    import torch
    B, Hq, N, D = q.shape
    shape = sa._Shape(B, Hq, k.shape[1], N, D)
    return sa.lib.sparse_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(host_mask._c()),
                                          ctypes.byref(p._c()), ctypes.byref(shape), scale, O.data_ptr(), L.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
def test_noalloc_matches_fwd_on_two_calls_in_a_row():
    """Both entry points run the same kernel on the same inputs with the same
    work plan, so their outputs agree bit for bit; the no-allocation output is
    also checked against the fp64 oracle at the parity bars."""
    import torch

    import oracle

    cases = [
        # (B, Hq, Hkv, N, D, pattern, block): ragged tail and GQA, then a strided pattern on 64-wide tiles
        (1, 4, 2, 1000, 128, sa.Pattern(window=200, sinks=4), 128),
        (2, 2, 2, 700, 64, sa.Pattern(window=40, stride=64, n_global=3), 64),
    ]
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    for i, (B, Hq, Hkv, N, D, p, block) in enumerate(cases):
        qh, kh, vh = synth.qkv(B, Hq, Hkv, N, D, seed=100 + i)
        q, k, v = dev(qh), dev(kh), dev(vh)
        scale = 1 / math.sqrt(D)
        host_mask = sa.build_block_mask(p, N, block)

        O_ref, L_ref = sa.fwd(q, k, v, host_mask.to_device("cuda"), p, scale=scale)
        assert sa.check_device() == sa.SA_OK

        O = torch.full_like(q, float("nan"))
        L = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device="cuda")
        rc = _noalloc(q, k, v, host_mask, p, scale, O, L)
        assert rc == sa.SA_OK, sa.status_string(rc)
        assert torch.equal(O, O_ref) and torch.equal(L, L_ref), i

        op = oracle.Pattern(window=p.window, sinks=p.sinks, stride=p.stride, n_global=p.n_global)
        Oo, Lo = oracle.attention(qh, kh, vh, op, scale)
        o_err = float(np.abs(O.float().cpu().numpy() - Oo).max())
        l_err = float(np.abs(L.cpu().numpy() - Lo).max())
        assert o_err <= O_TOL and l_err <= LSE_TOL, (i, o_err, l_err)


@pytest.mark.gpu
def test_noalloc_reports_a_device_timeout_and_recovers():
    """The wait limit and the skip-Q-load hook of sparse_attn_set_debug apply:
    the kernel's bounded waits expire (about 10 ms each), the call returns
    SA_ERR_DEVICE_TIMEOUT, and the next call on the same context is exact."""
    import torch

    B, Hq, Hkv, N, D = 1, 2, 2, 512, 128
    p = sa.Pattern(window=128, sinks=4)
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    q, k, v = (dev(a) for a in synth.qkv(B, Hq, Hkv, N, D, seed=7))
    host_mask = sa.build_block_mask(p, N, 128)
    O = torch.empty_like(q)
    L = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    try:
        sa.set_debug(sa.DEBUG_SKIP_Q_LOAD, 20_000_000)
        assert _noalloc(q, k, v, host_mask, p, 1 / math.sqrt(D), O, L) == sa.SA_ERR_DEVICE_TIMEOUT
    finally:
        sa.set_debug(0, 0)
    assert _noalloc(q, k, v, host_mask, p, 1 / math.sqrt(D), O, L) == sa.SA_OK
    O_ref, L_ref = sa.fwd(q, k, v, host_mask.to_device("cuda"), p, scale=1 / math.sqrt(D))
    assert sa.check_device() == sa.SA_OK
    assert torch.equal(O, O_ref) and torch.equal(L, L_ref)


@pytest.mark.gpu
def test_noalloc_at_the_largest_mask_its_scratch_holds():
    """T = 457 tiles per side (N = 58 496 at block 128, ragged by 37 rows), the
    largest mask the static scratch takes: bit for bit against sparse_attn_fwd
    and, on sampled rows, within the parity bars against the oracle."""
    import torch

    import oracle

    N, D = 457 * 128 - 37, 64
    p = sa.Pattern(window=500, sinks=4)
    q, k, v = synth.qkv(1, 2, 1, N, D, seed=12)
    t = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    Q, K, V = t(q), t(k), t(v)
    host_mask = sa.build_block_mask(p, N, 128)
    O_ref, L_ref = sa.fwd(Q, K, V, host_mask.to_device("cuda"), p, scale=1 / math.sqrt(D))
    O = torch.empty_like(Q)
    L = torch.empty_like(L_ref)
    assert _noalloc(Q, K, V, host_mask, p, 1 / math.sqrt(D), O, L) == sa.SA_OK
    torch.cuda.synchronize()
    assert torch.equal(O, O_ref) and torch.equal(L, L_ref)
    rows = np.unique(np.concatenate([np.arange(0, N, 128), np.arange(127, N, 128), [N - 1],
                                     np.random.default_rng(0).integers(0, N, 64)]))
    Oref, Lref = oracle.attention(q, k, v, oracle.Pattern(window=500, sinks=4), 1 / math.sqrt(D), rows=rows)
    Og = O.float().cpu().numpy()[:, :, rows]
    Lg = L.cpu().numpy()[:, :, rows]
    assert np.abs(Og - Oref).max() <= O_TOL and np.abs(Lg - Lref).max() <= LSE_TOL
