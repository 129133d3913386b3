"""Host-side checks of the C ABI (no GPU): the library loads, exports every
symbol the header declares, the pattern compiler agrees bit for bit with the
oracle's brute-force classifier, the pair counter with the oracle's count,
and argument errors come back as status codes."""
import ctypes
import os
import re

import numpy as np
import pytest

import block_sparse_attention_build_b200 as sa
import oracle
from synth.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            names |= set(re.findall(r"\b(sparse_attn_\w+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert "sparse_attn_fwd" in names and "sparse_attn_build_block_mask" in names
    for n in names:
        assert hasattr(sa.lib, n), n
    assert set(sa.EXPORTED) <= set(names)


def test_version_and_status_strings():
    assert sa.version() >= 100
    assert sa.status_string(0) == "ok"
    assert "timed out" in sa.status_string(sa.SA_ERR_DEVICE_TIMEOUT)


def opattern(p: sa.Pattern):
    return oracle.Pattern(window=p.window, sinks=p.sinks, stride=p.stride, n_global=p.n_global, causal=p.causal,
                          area=p.area, summary=p.summary)


SWEEP = [
    (sa.Pattern(window=w, sinks=s, stride=st, n_global=g), N, b)
    for (w, s, st, g) in [(1024, 4, 0, 0), (128, 4, 0, 0), (0, 0, 0, 0), (-1, 3, 0, 0), (63, 1, 0, 0),
                          (64, 0, 0, 0), (127, 128, 0, 0), (200, 130, 0, 0), (128, 0, 128, 16),
                          (10, 0, 7, 3), (-1, 0, 64, 0), (-1, 0, 1, 0), (5, 0, 200, 70), (300, 2, 3, 0),
                          (-1, 0, 0, 0), (100000, 0, 0, 0)]
    for N in (1, 63, 64, 65, 500, 1000, 1024)
    for b in (64, 128)
]


@pytest.mark.parametrize("p,N,b", SWEEP)
def test_block_mask_matches_oracle(p, N, b):
    m = sa.build_block_mask(p, N, b)
    c, i, f = oracle.block_mask(opattern(p), N, b)
    assert np.array_equal(m.counts, c) and np.array_equal(m.index, i) and np.array_equal(m.full, f)
    assert m.n_live == c.sum() and m.max_per_row == (c.max() if len(c) else 0)
    assert m.n_full == sum(int(f[r, : c[r]].sum()) for r in range(len(c)))


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_block_mask_workloads_match_oracle(name):
    w = WORKLOADS[name]
    p = sa.Pattern(**w.pattern_args())
    m = sa.build_block_mask(p, w.N, w.block)
    c, i, f = oracle.block_mask(opattern(p), w.N, w.block)
    assert np.array_equal(m.counts, c) and np.array_equal(m.index, i) and np.array_equal(m.full, f)
    assert sa.count_pairs(p, w.N) == oracle.count_pairs(opattern(p), w.N)


@pytest.mark.parametrize("p,N", [(p, N) for (p, N, b) in SWEEP if b == 64])
def test_pair_count_matches_oracle(p, N):
    assert sa.count_pairs(p, N) == oracle.count_pairs(opattern(p), N)


def test_empty_sequence():
    m = sa.build_block_mask(sa.Pattern(window=4), 0, 128)
    assert m.T == 0 and m.n_live == 0
    assert sa.count_pairs(sa.Pattern(window=4), 0) == 0


def test_builder_errors():
    with pytest.raises(sa.SparseAttnError) as e:
        sa.build_block_mask(sa.Pattern(window=4), 100, 32)
    assert e.value.status == sa.SA_ERR_UNSUPPORTED
    with pytest.raises(sa.SparseAttnError) as e:
        sa.build_block_mask(sa.Pattern(window=4, stride=2, causal=0), 100, 64)
    assert e.value.status == sa.SA_ERR_UNSUPPORTED
    with pytest.raises(sa.SparseAttnError) as e:
        sa.build_block_mask(sa.Pattern(window=-2), 100, 64)
    assert e.value.status == sa.SA_ERR_INVALID_ARG
    # capacity too small
    m = sa._BlockMask(1, 1, 0, 0, 0, 0, None, None, None)
    rc = sa.lib.sparse_attn_build_block_mask(ctypes.byref(sa.Pattern(window=4)._c()), 1000, 128, ctypes.byref(m))
    assert rc == sa.SA_ERR_BUFFER_TOO_SMALL


def test_fwd_argument_errors_without_gpu():
    """Checks that return before any CUDA call."""
    p = sa.Pattern(window=8)._c()
    m = sa._BlockMask(1, 1, 128, 1, 1, 0, 16, 16, 16)
    fake = 1 << 20  # never dereferenced: every case below fails validation first

    def call(shape, scale=0.125, mask=m, pat=p, ptr=fake):
        return sa.lib.sparse_attn_fwd(ptr, ptr, ptr, ctypes.byref(mask), ctypes.byref(pat),
                                      ctypes.byref(sa._Shape(*shape)), scale, ptr, ptr, None)

    assert call((1, 2, 2, 100, 96)) == sa.SA_ERR_UNSUPPORTED          # D
    assert call((1, 2, 2, 100, 128), scale=0.0) == sa.SA_ERR_INVALID_ARG
    assert call((1, 2, 2, 100, 128), scale=float("nan")) == sa.SA_ERR_INVALID_ARG
    assert call((1, 3, 2, 100, 128)) == sa.SA_ERR_UNSUPPORTED         # Hq % Hkv
    assert call((1, 2, 2, 1000, 128)) == sa.SA_ERR_MASK_MISMATCH      # T != ceil(N / block)
    assert call((-1, 2, 2, 100, 128)) == sa.SA_ERR_INVALID_ARG
    assert call((1, 2, 2, 100, 128), ptr=fake + 8) == sa.SA_ERR_MISALIGNED
    assert call((0, 2, 2, 100, 128)) == sa.SA_OK                      # nothing to compute
    assert call((1, 2, 2, 0, 128)) == sa.SA_OK
    bad = sa.Pattern(window=8, stride=4, causal=0)._c()
    assert call((1, 2, 2, 100, 128), pat=bad) == sa.SA_ERR_UNSUPPORTED
    ws = ctypes.c_size_t(0)
    assert sa.lib.sparse_attn_fwd_host_workspace(ctypes.byref(sa._Shape(1, 2, 1, 100, 64)), ctypes.byref(ws)) == 0
    assert ws.value >= 2 * (2 * 100 * 64 * 2) + 2 * (100 * 64 * 2) + 2 * 100 * 4


def test_fwd_heads_argument_errors_without_gpu():
    """Per-head entry point: checks that return before any CUDA call."""
    p = sa.Pattern(window=8)._c()
    p2 = sa.Pattern(window=4, stride=16)._c()
    m = sa._BlockMask(1, 1, 128, 1, 1, 0, 16, 16, 16)
    m64 = sa._BlockMask(2, 2, 64, 1, 1, 0, 16, 16, 16)
    fake = 1 << 20  # never dereferenced: every case below fails validation first

    def call(shape, heads, masks=(m, m), pats=(p, p2), n=None, ptr=fake):
        n = len(pats) if n is None else n
        cm = (sa._BlockMask * len(masks))(*masks)
        cp = (sa._Pattern * len(pats))(*pats)
        ch = (ctypes.c_int32 * max(len(heads), 1))(*heads)
        return sa.lib.sparse_attn_fwd_heads(ptr, ptr, ptr, cm, cp, n, ch if heads is not None else None,
                                            ctypes.byref(sa._Shape(*shape)), 0.125, ptr, ptr, None)

    assert call((1, 2, 2, 100, 128), [0, 1], n=0) == sa.SA_ERR_INVALID_ARG          # no pattern
    assert call((1, 2, 2, 100, 128), [0, 1], n=9) == sa.SA_ERR_INVALID_ARG          # more than 8
    assert call((1, 2, 2, 100, 128), [0, 2]) == sa.SA_ERR_INVALID_ARG               # index out of range
    assert call((1, 2, 2, 100, 128), [0, -1]) == sa.SA_ERR_INVALID_ARG
    assert call((1, 2, 2, 100, 128), [0, 1], masks=(m, m64)) == sa.SA_ERR_MASK_MISMATCH  # blocks differ
    assert call((1, 300, 300, 100, 128), [0] * 300) == sa.SA_ERR_UNSUPPORTED         # more than 256 heads
    bad = sa.Pattern(window=8, stride=4, causal=0)._c()
    assert call((1, 2, 2, 100, 128), [0, 1], pats=(p, bad)) == sa.SA_ERR_UNSUPPORTED
    assert call((1, 2, 2, 100, 128), [0, 1], ptr=fake + 8) == sa.SA_ERR_MISALIGNED
    assert call((0, 2, 2, 100, 128), [0, 1]) == sa.SA_OK                             # nothing to compute
    rc = sa.lib.sparse_attn_fwd_heads(fake, fake, fake, (sa._BlockMask * 1)(m), (sa._Pattern * 1)(p), 1, None,
                                      ctypes.byref(sa._Shape(1, 2, 2, 100, 128)), 0.125, fake, fake, None)
    assert rc == sa.SA_ERR_INVALID_ARG                                               # no head table


def transpose_of_oracle(p, N, b):
    """The oracle's brute-force classification, read column by column."""
    c, i, f = oracle.block_mask(opattern(p), N, b)
    T = len(c)
    tc = np.zeros(T, dtype=np.int32)
    ti = np.full((T, T), -1, dtype=np.int32)
    tf = np.zeros((T, T), dtype=np.uint8)
    for r in range(T):
        for e in range(c[r]):
            col = i[r, e]
            ti[col, tc[col]] = r
            tf[col, tc[col]] = f[r, e]
            tc[col] += 1
    return tc, ti, tf


@pytest.mark.parametrize("p,N,b", SWEEP[::3])
def test_transposed_mask_matches_oracle(p, N, b):
    m = sa.transpose_block_mask(sa.build_block_mask(p, N, b))
    tc, ti, tf = transpose_of_oracle(p, N, b)
    assert np.array_equal(m.counts, tc) and np.array_equal(m.index, ti) and np.array_equal(m.full, tf)
    assert m.n_live == tc.sum() and m.block == b


def test_transpose_errors():
    good = sa.build_block_mask(sa.Pattern(window=300, sinks=4), 1000, 128)
    bad_index = good.index.copy()
    bad_index[3, 0] = 99
    broken = sa.BlockMask(good.counts, bad_index, good.full, 128, good.n_live, good.n_full, good.max_per_row, 1000)
    with pytest.raises(sa.SparseAttnError) as e:
        sa.transpose_block_mask(broken)
    assert e.value.status == sa.SA_ERR_INVALID_ARG
    small = sa._BlockMask(2, 2, 0, 0, 0, 0, None, None, None)
    rc = sa.lib.sparse_attn_transpose_block_mask(ctypes.byref(good._c()), ctypes.byref(small))
    assert rc == sa.SA_ERR_BUFFER_TOO_SMALL


def test_bwd_argument_errors_without_gpu():
    """Checks that return before any CUDA call."""
    p = sa.Pattern(window=8)._c()
    m = sa._BlockMask(1, 1, 128, 1, 1, 0, 16, 16, 16)
    fake = 1 << 20
    ws_ok = sa.bwd_workspace_bytes(1, 2, 2, 100, 128)

    def call(shape, scale=0.125, mask=m, pat=p, ptr=fake, ws=fake, ws_bytes=ws_ok):
        return sa.lib.sparse_attn_bwd(ptr, ptr, ptr, ptr, ptr, ptr, ctypes.byref(mask), ctypes.byref(pat),
                                      ctypes.byref(sa._Shape(*shape)), scale, ptr, ptr, ptr, ws, ws_bytes, None)

    assert call((1, 2, 2, 100, 96)) == sa.SA_ERR_UNSUPPORTED                       # D
    assert call((1, 2, 2, 100, 128), scale=0.0) == sa.SA_ERR_INVALID_ARG
    assert call((1, 3, 2, 100, 128)) == sa.SA_ERR_UNSUPPORTED                      # Hq % Hkv
    assert call((1, 2, 2, 1000, 128)) == sa.SA_ERR_MASK_MISMATCH                   # T != ceil(N / 128)
    m64 = sa._BlockMask(2, 2, 64, 1, 1, 0, 16, 16, 16)
    assert call((1, 2, 2, 100, 128), mask=m64) == sa.SA_ERR_UNSUPPORTED            # block 64
    assert call((1, 2, 2, 100, 128), ptr=fake + 8) == sa.SA_ERR_MISALIGNED
    assert call((1, 2, 2, 100, 128), ws=fake + 16) == sa.SA_ERR_MISALIGNED         # workspace 256-aligned
    assert call((1, 2, 2, 100, 128), ws_bytes=ws_ok - 1) == sa.SA_ERR_BUFFER_TOO_SMALL
    assert call((0, 2, 2, 100, 128)) == sa.SA_OK
    bad = sa.Pattern(window=8, stride=4, causal=0)._c()
    assert call((1, 2, 2, 100, 128), pat=bad) == sa.SA_ERR_UNSUPPORTED
    rows = 1 * 2 * 100
    assert ws_ok >= 2 * rows * 4 + rows * 128 * 4


GENERAL = [
    (sa.Pattern(window=w, sinks=s, n_global=g, causal=c, area=a), N, b)
    for (w, s, g, c, a) in [(37, 0, 0, 0, 0), (-1, 0, 0, 0, 400), (-1, 0, 0, 0, 100), (5, 3, 0, 0, 0),
                            (2, 0, 4, 0, 0), (-1, 2, 0, 0, 77), (20, 0, 0, 1, 64), (-1, 0, 0, 1, 400),
                            (300, 1, 2, 0, 130), (0, 0, 0, 0, 1), (-1, 0, 0, 0, 0), (5000, 0, 0, 0, 0)]
    for N in (1, 100, 500, 1000, 1600)
    for b in (64, 128)
] + [
    # the fixed pattern: blocks of `area` plus the last `summary` positions of every block
    (sa.Pattern(window=w, sinks=s, causal=c, area=a, summary=m), N, b)
    for (w, s, c, a, m) in [(-1, 0, 1, 128, 16), (-1, 0, 1, 100, 10), (-1, 0, 0, 64, 8), (3, 2, 1, 50, 7),
                            (-1, 0, 1, 16, 16), (-1, 0, 1, 40, 100), (10, 0, 0, 33, 1)]
    for N in (1, 300, 1000)
    for b in (64, 128)
]


@pytest.mark.parametrize("p,N,b", GENERAL)
def test_general_block_mask_matches_oracle(p, N, b):
    m = sa.build_block_mask(p, N, b)
    c, i, f = oracle.block_mask(opattern(p), N, b)
    assert np.array_equal(m.counts, c) and np.array_equal(m.index, i) and np.array_equal(m.full, f)
    assert sa.count_pairs(p, N) == oracle.count_pairs(opattern(p), N)
    t = sa.transpose_block_mask(m)
    tc, ti, tf = transpose_of_oracle(p, N, b)
    assert np.array_equal(t.counts, tc) and np.array_equal(t.index, ti) and np.array_equal(t.full, tf)


def test_area_attention_printed_pair_count():
    assert sa.count_pairs(sa.Pattern(window=-1, causal=0, area=400), 1600) == 640000


def test_general_pattern_errors():
    for p, rc in [(sa.Pattern(window=4, stride=8, causal=0), sa.SA_ERR_UNSUPPORTED),
                  (sa.Pattern(window=4, stride=8, area=64), sa.SA_ERR_UNSUPPORTED),
                  (sa.Pattern(window=4, causal=2), sa.SA_ERR_UNSUPPORTED),
                  (sa.Pattern(window=4, area=-1), sa.SA_ERR_INVALID_ARG),
                  (sa.Pattern(window=4, summary=2), sa.SA_ERR_INVALID_ARG),       # summary needs area
                  (sa.Pattern(window=4, area=8, summary=-1), sa.SA_ERR_INVALID_ARG)]:
        with pytest.raises(sa.SparseAttnError) as e:
            sa.build_block_mask(p, 100, 64)
        assert e.value.status == rc
        with pytest.raises(sa.SparseAttnError) as e:
            sa.count_pairs(p, 100)
        assert e.value.status == rc
    # the forward and backward entry points check the same before any CUDA call
    m = sa._BlockMask(1, 1, 128, 1, 1, 0, 16, 16, 16)
    fake = 1 << 20
    bad = sa.Pattern(window=4, stride=8, causal=0)._c()
    shape = sa._Shape(1, 2, 2, 100, 128)
    assert sa.lib.sparse_attn_fwd(fake, fake, fake, ctypes.byref(m), ctypes.byref(bad), ctypes.byref(shape), 0.1,
                                  fake, fake, None) == sa.SA_ERR_UNSUPPORTED
    assert sa.lib.sparse_attn_bwd(fake, fake, fake, fake, fake, fake, ctypes.byref(m), ctypes.byref(bad),
                                  ctypes.byref(shape), 0.1, fake, fake, fake, fake, 1 << 30, None) == sa.SA_ERR_UNSUPPORTED
    area = sa.Pattern(window=-1, causal=0, area=64)._c()
    assert sa.lib.sparse_attn_fwd_noalloc(fake, fake, fake, ctypes.byref(m), ctypes.byref(area), ctypes.byref(shape),
                                          0.1, fake, fake, None) == sa.SA_ERR_UNSUPPORTED
    big = sa._Shape(1, 300, 300, 100, 128)  # general forms use the pattern-table kernel: Hq <= 256
    assert sa.lib.sparse_attn_fwd(fake, fake, fake, ctypes.byref(m), ctypes.byref(area), ctypes.byref(big), 0.1,
                                  fake, fake, None) == sa.SA_ERR_UNSUPPORTED


def test_fixed_pattern_pair_count_closed_form():
    # causal: q mod A + 1 keys of the own block, plus c summary keys in every earlier block
    for N, A, c in [(1024, 128, 16), (1000, 100, 10), (333, 64, 1)]:
        assert sa.count_pairs(sa.Pattern(window=-1, area=A, summary=c), N) == sum(
            q % A + 1 + (q // A) * c for q in range(N))


STRIDE_PLANS = [
    (sa.Pattern(window=8, stride=8, n_global=2), 128, 64),      # the strided-global shape, scaled down
    (sa.Pattern(window=5, stride=4, sinks=3), 192, 64),
    (sa.Pattern(window=-1, stride=6), 192, 64),                 # stride only
    (sa.Pattern(window=13, stride=4, n_global=9), 256, 64),     # global wider than the stride
    (sa.Pattern(window=2, stride=16, sinks=1), 256, 64),        # groups of 16 inside a tile
    (sa.Pattern(window=128, stride=128, n_global=16), 1024, 64),  # groups of 8 tokens
    (sa.Pattern(window=40, stride=2, sinks=4), 256, 128),       # groups of 128: one tile each
]


@pytest.mark.parametrize("p,N,b", STRIDE_PLANS)
def test_stride_plan_matches_brute_force(p, N, b):
    pass1, pass2 = sa.stride_plan(p, N, b)
    p1 = sa.Pattern(window=p.window, sinks=p.sinks, n_global=p.n_global)
    c, i, f = oracle.block_mask(opattern(p1), N, b)
    assert np.array_equal(pass1.counts, c) and np.array_equal(pass1.index, i) and np.array_equal(pass1.full, f)
    # pass 2 must hold exactly the pairs of the whole pattern that pass 1 lacks, in the grouped order
    s, n = p.stride, N // p.stride
    pos = lambda t: (t % s) * n + t // s
    full_p, base_p = opattern(p), opattern(p1)
    grid = np.zeros((N, N), dtype=bool)
    for q in range(N):
        for kv in range(q + 1):
            if oracle.allowed(full_p, q, kv) and not oracle.allowed(base_p, q, kv):
                grid[pos(q), pos(kv)] = True
    T = -(-N // b)
    for ti in range(T):
        rows = grid[ti * b:(ti + 1) * b]
        js = [tj for tj in range(T) if rows[:, tj * b:(tj + 1) * b].any()]
        assert pass2.counts[ti] == len(js)
        assert list(pass2.index[ti, :len(js)]) == js and all(pass2.index[ti, len(js):] == -1)
        fl = [int(rows[:, tj * b:(tj + 1) * b].all()) for tj in js]
        assert list(pass2.full[ti, :len(js)]) == fl
    assert grid.sum() + oracle.count_pairs(base_p, N) == oracle.count_pairs(full_p, N)


def test_stride_plan_errors():
    for p, N, rc in [(sa.Pattern(window=4), 64, sa.SA_ERR_UNSUPPORTED),                 # no stride
                     (sa.Pattern(window=4, stride=6), 64, sa.SA_ERR_UNSUPPORTED),       # N not a multiple
                     (sa.Pattern(window=4, stride=4, causal=0), 64, sa.SA_ERR_UNSUPPORTED)]:
        with pytest.raises(sa.SparseAttnError) as e:
            sa.stride_plan(p, N, 64)
        assert e.value.status == rc
    m = sa._BlockMask(1, 1, 128, 1, 1, 0, 16, 16, 16)
    fake = 1 << 20
    shape = sa._Shape(1, 2, 2, 96, 128)
    good = sa.Pattern(window=8, stride=8)._c()
    call = lambda pat, ws=fake, nbytes=1 << 30, ptr=fake: sa.lib.sparse_attn_fwd_stride(
        ptr, ptr, ptr, ctypes.byref(m), ctypes.byref(m), ctypes.byref(pat), ctypes.byref(shape), 0.1, ptr, ptr, ws,
        nbytes, None)
    assert call(sa.Pattern(window=8)._c()) == sa.SA_ERR_UNSUPPORTED
    assert call(sa.Pattern(window=8, stride=7)._c()) == sa.SA_ERR_UNSUPPORTED  # 96 % 7
    assert call(good, ws=fake + 16) == sa.SA_ERR_MISALIGNED
    assert call(good, nbytes=100) == sa.SA_ERR_BUFFER_TOO_SMALL
    assert call(good, ptr=fake + 8) == sa.SA_ERR_MISALIGNED


def test_bwd_heads_argument_errors_without_gpu():
    p = sa.Pattern(window=8)._c()
    p2 = sa.Pattern(window=4, stride=16)._c()
    m = sa._BlockMask(1, 1, 128, 1, 1, 0, 16, 16, 16)
    m64 = sa._BlockMask(2, 2, 64, 1, 1, 0, 16, 16, 16)
    fake = 1 << 20
    ws = sa.bwd_workspace_bytes(1, 2, 2, 100, 128)

    def call(shape, heads, masks=(m, m), pats=(p, p2), n=None):
        n = len(pats) if n is None else n
        cm = (sa._BlockMask * len(masks))(*masks)
        cp = (sa._Pattern * len(pats))(*pats)
        ch = (ctypes.c_int32 * max(len(heads), 1))(*heads)
        return sa.lib.sparse_attn_bwd_heads(fake, fake, fake, fake, fake, fake, cm, cp, n, ch,
                                            ctypes.byref(sa._Shape(*shape)), 0.125, fake, fake, fake, fake, ws, None)

    assert call((1, 2, 2, 100, 128), [0, 1], n=0) == sa.SA_ERR_INVALID_ARG
    assert call((1, 2, 2, 100, 128), [0, 1], n=9) == sa.SA_ERR_INVALID_ARG
    assert call((1, 2, 2, 100, 128), [0, 2]) == sa.SA_ERR_INVALID_ARG
    assert call((1, 2, 2, 100, 128), [0, 1], masks=(m, m64)) == sa.SA_ERR_UNSUPPORTED   # block 64
    assert call((1, 300, 300, 100, 128), [0] * 300) == sa.SA_ERR_UNSUPPORTED
    bad = sa.Pattern(window=8, stride=4, causal=0)._c()
    assert call((1, 2, 2, 100, 128), [0, 1], pats=(p, bad)) == sa.SA_ERR_UNSUPPORTED
    assert call((0, 2, 2, 100, 128), [0, 1]) == sa.SA_OK
    rc = sa.lib.sparse_attn_bwd_heads(fake, fake, fake, fake, fake, fake, (sa._BlockMask * 1)(m),
                                      (sa._Pattern * 1)(p), 1, None, ctypes.byref(sa._Shape(1, 2, 2, 100, 128)),
                                      0.125, fake, fake, fake, fake, ws, None)
    assert rc == sa.SA_ERR_INVALID_ARG


def _malformed_masks(N=1000, block=128):
    """A well-formed host mask and variants that break one rule each."""
    good = sa.build_block_mask(sa.Pattern(window=300, sinks=4), N, block)

    def variant(edit):
        c, i, f = good.counts.copy(), good.index.copy(), good.full.copy()
        edit(c, i, f)
        return sa.BlockMask(c, i, f, good.block, good.n_live, good.n_full, good.max_per_row, N)

    T = good.T
    bad = {
        "count above T": variant(lambda c, i, f: c.__setitem__(2, T + 1)),
        "negative count": variant(lambda c, i, f: c.__setitem__(3, -1)),
        "index past T": variant(lambda c, i, f: i.__setitem__((5, c[5] - 1), T)),
        "negative index": variant(lambda c, i, f: i.__setitem__((4, 0), -1)),
        "not ascending": variant(lambda c, i, f: i.__setitem__((6, 1), i[6, 0])),
        "flag not 0 or 1": variant(lambda c, i, f: f.__setitem__((7, 0), 2)),
    }
    return good, bad


def test_host_mask_checked_before_device_work():
    """sparse_attn_fwd_host and sparse_attn_fwd_noalloc read the block mask on
    the host: a malformed one comes back as SA_ERR_INVALID_ARG before any CUDA
    call (the tensor pointers below are never dereferenced)."""
    N, D = 1000, 128
    good, bad = _malformed_masks(N)
    p = sa.Pattern(window=300, sinks=4)._c()
    shape = sa._Shape(1, 2, 2, N, D)
    fake = 1 << 20
    ws = ctypes.c_size_t(0)
    assert sa.lib.sparse_attn_fwd_host_workspace(ctypes.byref(shape), ctypes.byref(ws)) == 0
    for name, m in bad.items():
        cm = m._c()
        rc = sa.lib.sparse_attn_fwd_host(fake, fake, fake, ctypes.byref(cm), ctypes.byref(p), ctypes.byref(shape),
                                         0.088, fake, fake, fake, ws.value, None)
        assert rc == sa.SA_ERR_INVALID_ARG, (name, rc)
        rc = sa.lib.sparse_attn_fwd_noalloc(fake, fake, fake, ctypes.byref(cm), ctypes.byref(p), ctypes.byref(shape),
                                            0.088, fake, fake, None)
        assert rc == sa.SA_ERR_INVALID_ARG, (name, rc)
    # a short workspace and a misplaced mask are refused the same way
    cm = good._c()
    rc = sa.lib.sparse_attn_fwd_host(fake, fake, fake, ctypes.byref(cm), ctypes.byref(p), ctypes.byref(shape), 0.088,
                                     fake, fake, fake, ws.value - 1, None)
    assert rc == sa.SA_ERR_BUFFER_TOO_SMALL
    other = sa.build_block_mask(sa.Pattern(window=300, sinks=4), 2 * N, 128)._c()
    rc = sa.lib.sparse_attn_fwd_host(fake, fake, fake, ctypes.byref(other), ctypes.byref(p), ctypes.byref(shape),
                                     0.088, fake, fake, fake, ws.value, None)
    assert rc == sa.SA_ERR_MASK_MISMATCH


def test_host_workspace_covers_the_mask_copy():
    """The host-buffer workspace holds Q, K, V, O, LSE and a copy of a mask of
    ceil(N / 64) tiles per side."""
    B, Hq, Hkv, N, D = 2, 4, 2, 1000, 64
    ws = ctypes.c_size_t(0)
    assert sa.lib.sparse_attn_fwd_host_workspace(ctypes.byref(sa._Shape(B, Hq, Hkv, N, D)), ctypes.byref(ws)) == 0
    T = -(-N // 64)
    need = 2 * B * Hq * N * D * 2 + 2 * B * Hkv * N * D * 2 + B * Hq * N * 4 + T * 4 + 5 * T * T
    assert need <= ws.value <= need + 8 * 256


def test_more_tiles_than_the_kernel_takes_is_refused_without_gpu():
    """4097 tiles per side (one past the step lists' 12-bit tile indices) is
    SA_ERR_UNSUPPORTED before any CUDA call; 4096 passes the check (the fake
    pointers then stop it at alignment, still before any CUDA call)."""
    p = sa.Pattern(window=8)._c()
    fake = 1 << 20
    for T, want in ((4097, sa.SA_ERR_UNSUPPORTED), (4096, sa.SA_ERR_MISALIGNED)):
        m = sa._BlockMask(T, T, 128, 1, 1, 0, fake, fake, fake)
        shape = sa._Shape(1, 1, 1, T * 128, 128)
        rc = sa.lib.sparse_attn_fwd(fake + 8, fake, fake, ctypes.byref(m), ctypes.byref(p), ctypes.byref(shape),
                                    0.1, fake, fake, None)
        assert rc == want, (T, rc)


def test_headline_tile_lists_are_a_diagonal_band_plus_the_sink_column():
    """The headline pattern's picture ("Sparse Attention" glossary page, section
    "Ein Muster in Einsparungen verwandeln"): every query tile lists kv tile 0
    (the sinks) and the tiles from 8 before the diagonal up to it (a 1024-token
    window is 8 tiles of 128, and q - kv <= 1024 reaches one more), nothing else;
    only the diagonal tiles and the band's far edge are partial."""
    m = sa.build_block_mask(sa.Pattern(window=1024, sinks=4), 8192, 128)
    for i in range(m.T):
        want = sorted({0} | set(range(max(0, i - 8), i + 1)))
        assert list(m.index[i, : m.counts[i]]) == want, i
        full = {int(j) for j, f in zip(m.index[i, : m.counts[i]], m.full[i, : m.counts[i]]) if f}
        # full: the tiles strictly inside the band (1 <= i - j <= 7)
        assert full == set(range(max(0, i - 7), i)), i


def test_binding_refuses_a_mask_in_the_wrong_memory():
    """Host-side calls take numpy masks, device calls a copy on the tensors'
    device: a mask in the other memory is a TypeError in the binding, before
    the library could read host addresses on the device or the reverse."""
    import torch
    m = sa.build_block_mask(sa.Pattern(window=100, sinks=4), 1000, 128)
    as_torch = sa.BlockMask(*(torch.from_numpy(a) for a in (m.counts, m.index, m.full)),
                            m.block, m.n_live, m.n_full, m.max_per_row, m.N)
    assert m.on_host and not as_torch.on_host
    with pytest.raises(TypeError, match="host block mask"):
        sa.transpose_block_mask(as_torch)
    with pytest.raises(TypeError, match="host block mask"):
        sa._host_masks("fwd_noalloc", as_torch)
    for mask in (m, as_torch):  # numpy arrays, or torch tensors in host memory
        with pytest.raises(TypeError, match="tensors' device"):
            sa._device_masks("fwd", torch.device("cuda", 0), mask)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No fallback: without the built library the binding refuses to load."""
    monkeypatch.setattr(sa, "LIB_PATH", str(tmp_path / "libsparse_attn.so"))
    with pytest.raises(ImportError, match="missing"):
        sa._load()


def test_product_and_oracle_share_no_code():
    """The package (binding and CUDA sources) never names the oracle, and the
    oracle never names the package, its library or its headers."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "block_sparse_attention_build_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert re.search(r"\boracle\b", text) is None, f
    for f in os.listdir(os.path.join(root, "oracle")):
        if f.endswith((".py", ".c", ".h")):
            text = open(os.path.join(root, "oracle", f), encoding="utf-8").read()
            for name in ("block_sparse_attention_build_b200", "sparse_attn.h", "libsparse_attn", "sparse_attn_"):
                assert name not in text, (f, name)
