"""Pins for the CPU oracle, checked against facts that do not come from the
oracle itself: the figure the pages print, closed forms derived from the
pattern definitions, brute force on tiny inputs, identities of the softmax and
library routines (torch's scaled_dot_product_attention in fp64)."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import Pattern

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split()
                vals[k] = v
    return vals


def live_and_full(counts, full):
    live = int(counts.sum())
    nfull = int(sum(full[i, : counts[i]].sum() for i in range(len(counts))))
    return live, nfull


# ----------------------------------------------------------------------------
# The printed figure.

def test_printed_sparsity_window_sinks():
    g = read_golden("sparsity_window_sinks.txt")
    N, w, s, b = int(g["seq_len"]), int(g["window"]), int(g["sinks"]), int(g["block"])
    counts, index, full = oracle.block_mask(Pattern(window=w, sinks=s), N, b)
    T = N // b
    sparsity = 100.0 * (1.0 - counts.sum() / (T * T))
    assert f"{sparsity:.2f}" == g["sparsity_percent"]
    # the picture the page describes: a left column for the sinks, a diagonal band
    for i in range(T):
        row = index[i, : counts[i]]
        assert row[0] == 0 and row[-1] == i


def test_prototype_output_shape():
    g = read_golden("prototype_shape.txt")
    n, d = int(g["n"]), int(g["d"])
    q, k, v = synth.qkv(1, 1, 1, n, d, seed=3)
    O, LSE = oracle.attention(q, k, v, Pattern(window=int(g["window_exclusive"]) - 1), 1 / math.sqrt(d))
    assert O.shape[2:] == (int(g["out_rows"]), int(g["out_cols"]))


# ----------------------------------------------------------------------------
# Closed forms, derived from the definitions rather than counted.

def closed_live_window_sinks(T, w, b, sinks):
    """Row i of tiles reaches back K = ceil(w / b) tiles, plus tile 0 when sinks
    exist and the band does not already reach it."""
    K = -(-w // b)
    live = sum(min(i, K) + 1 for i in range(T))
    if sinks > 0:
        live += max(0, T - 1 - K)
    return live


def closed_full_window_sinks(T, w, b):
    """Tile (i, j < i) is full when its largest distance (i - j + 1) b - 1 is <= w
    (sinks < b, so the sink column never fills a tile on its own)."""
    F = (w + 1) // b - 1
    return sum(max(0, min(i, F)) for i in range(T))


def closed_pairs_window_sinks(N, w, sinks):
    return sum(min(q, w) + 1 + min(sinks, max(0, q - w)) for q in range(N))


def closed_row_count_strided(q, l, s, G):
    """|A(q)| for a causal band of width l, every s-th prior token and G global
    tokens, by inclusion-exclusion over distances delta = q - kv in [0, q]."""
    if q < G:
        return q + 1
    n = min(q, l) + 1                          # band: delta in [0, min(q, l)]
    if q > l:
        n += q // s - l // s                   # multiples of s in (l, q]
    lo = max(q - G + 1, l + 1)                 # global columns kv < G: delta in [q-G+1, q]
    if lo <= q:
        mult = q // s - (lo - 1) // s          # multiples of s in [lo, q], already counted
        n += (q - lo + 1) - mult
    return n


@pytest.mark.parametrize("N,w,sinks,b", [
    (8192, 1024, 4, 128), (512, 128, 4, 64), (32768, 4096, 0, 128), (16384, 128, 4, 128),
    (1000, 100, 3, 64), (777, 0, 1, 64), (640, 300, 0, 128), (2048, 5000, 0, 128),
])
def test_tile_counts_closed_form(N, w, sinks, b):
    counts, _, full = oracle.block_mask(Pattern(window=w, sinks=sinks), N, b)
    T = -(-N // b)
    live, nfull = live_and_full(counts, full)
    assert live == closed_live_window_sinks(T, w, b, sinks)
    if N % b == 0:
        assert nfull == closed_full_window_sinks(T, w, b)


@pytest.mark.parametrize("N,w,sinks", [(512, 128, 4), (8192, 1024, 4), (3000, 17, 5), (100, 200, 0)])
def test_pair_count_closed_form(N, w, sinks):
    assert oracle.count_pairs(Pattern(window=w, sinks=sinks), N) == closed_pairs_window_sinks(N, w, sinks)


@pytest.mark.parametrize("N,l,s,G", [(16384, 128, 128, 16), (1000, 10, 7, 3), (300, 0, 5, 0), (257, 64, 64, 70)])
def test_pair_count_strided_closed_form(N, l, s, G):
    expect = sum(closed_row_count_strided(q, l, s, G) for q in range(N))
    assert oracle.count_pairs(Pattern(window=l, stride=s, n_global=G), N) == expect


def test_dense_counts():
    # Window wider than the sequence and no sinks: the causal triangle, N(N+1)/2 pairs,
    # and every tile on or below the diagonal is live.
    N, b = 1024, 128
    p = Pattern(window=N)
    assert oracle.count_pairs(p, N) == N * (N + 1) // 2
    counts, _, full = oracle.block_mask(p, N, b)
    T = N // b
    live, nfull = live_and_full(counts, full)
    assert live == T * (T + 1) // 2 and nfull == T * (T - 1) // 2


# ----------------------------------------------------------------------------
# Brute force on tiny inputs: the allowed set written as a union of the rule
# sets of the pages, tiled by hand.

def rule_sets(N, q, p: Pattern):
    causal = set(range(0, q + 1))
    s = set()
    if p.window >= 0:
        s |= set(range(max(0, q - p.window), q + 1))
    s |= set(range(0, min(p.sinks, N)))
    if p.stride > 0:
        s |= set(range(q, -1, -p.stride))
    s |= set(range(0, min(p.n_global, N)))
    if q < p.n_global:
        s |= set(range(0, N))
    out = s & causal
    if p.global_rows_see_all and q < p.n_global:
        out = set(range(N))
    return out


TINY = [
    (Pattern(window=3, sinks=2), 37, 8),
    (Pattern(window=0), 20, 4),
    (Pattern(window=5, stride=4, n_global=2), 41, 8),
    (Pattern(window=-1, stride=3), 30, 8),
    (Pattern(window=2, n_global=5, global_rows_see_all=1), 33, 8),
    (Pattern(window=-1, sinks=0), 17, 4),
    (Pattern(window=6, sinks=9), 50, 16),
    (Pattern(window=30, sinks=2), 37, 8),
]


@pytest.mark.parametrize("p,N,b", TINY)
def test_block_mask_brute_force_tiny(p, N, b):
    sets = [rule_sets(N, q, p) for q in range(N)]
    for q in range(N):
        for kv in range(N):
            assert oracle.allowed(p, q, kv) == (kv in sets[q])
    T = -(-N // b)
    counts, index, full = oracle.block_mask(p, N, b)
    for i in range(T):
        row_j, row_f = [], []
        for j in range(T):
            qs = range(i * b, min(N, (i + 1) * b))
            ks = range(j * b, min(N, (j + 1) * b))
            n = sum(1 for q in qs for kv in ks if kv in sets[q])
            if n:
                row_j.append(j)
                row_f.append(int(n == len(qs) * len(ks)))
        assert counts[i] == len(row_j)
        assert list(index[i, : counts[i]]) == row_j and all(index[i, counts[i]:] == -1)
        assert list(full[i, : counts[i]]) == row_f and all(full[i, counts[i]:] == 0)
    assert oracle.count_pairs(p, N) == sum(len(s) for s in sets)


# ----------------------------------------------------------------------------
# Softmax identities and library routines.

def to_f64(bits):
    return torch.from_numpy(synth.bf16_bits_to_float(bits)).double()


def test_dense_causal_equals_sdpa():
    B, Hq, Hkv, N, D = 2, 4, 2, 130, 32
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=11)
    scale = 1 / math.sqrt(D)
    O, LSE = oracle.attention(q, k, v, Pattern(window=N), scale)
    kt = to_f64(k).repeat_interleave(Hq // Hkv, dim=1)
    vt = to_f64(v).repeat_interleave(Hq // Hkv, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(to_f64(q), kt, vt, is_causal=True, scale=scale)
    assert np.abs(O - ref.numpy()).max() < 1e-12
    s = to_f64(q) @ kt.transpose(-1, -2) * scale
    s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    assert np.abs(LSE - torch.logsumexp(s, dim=-1).numpy()).max() < 1e-12


@pytest.mark.parametrize("p,N", [(Pattern(window=9, sinks=3), 70), (Pattern(window=4, stride=6, n_global=3), 65),
                                 (Pattern(window=2, n_global=4, global_rows_see_all=1), 40)])
def test_masked_equals_sdpa_with_explicit_mask(p, N):
    B, Hq, Hkv, D = 1, 4, 1, 16
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=5)
    scale = 0.37
    O, LSE = oracle.attention(q, k, v, p, scale)
    mask = torch.zeros(N, N, dtype=torch.bool)
    for qi in range(N):
        mask[qi, sorted(rule_sets(N, qi, p))] = True
    kt = to_f64(k).repeat_interleave(Hq // Hkv, dim=1)
    vt = to_f64(v).repeat_interleave(Hq // Hkv, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(to_f64(q), kt, vt, attn_mask=mask, scale=scale)
    assert np.abs(O - ref.numpy()).max() < 1e-12


def test_zero_query_gives_log_count_and_mean():
    # Q = 0: every allowed key gets weight 1/|A(q)|, so LSE = ln |A(q)| and O is the mean of V over A(q).
    N, D, w, sinks = 300, 16, 40, 4
    q = np.zeros((1, 2, N, D), dtype=np.uint16)
    _, k, v = synth.qkv(1, 2, 2, N, D, seed=9)
    O, LSE = oracle.attention(q, k, v, Pattern(window=w, sinks=sinks), 0.125)
    cnt = np.array([min(r, w) + 1 + min(sinks, max(0, r - w)) for r in range(N)])
    assert np.abs(LSE - np.log(cnt)[None, None]).max() < 1e-12
    vf = synth.bf16_bits_to_float(v).astype(np.float64)
    for r in (0, 3, 41, 45, 299):
        keys = sorted(set(range(max(0, r - w), r + 1)) | set(range(min(sinks, r + 1))))
        assert np.abs(O[:, :, r] - vf[:, :, keys].mean(axis=2)).max() < 1e-12


def test_zero_query_strided_log_count():
    N, D, l, s, G = 400, 8, 16, 16, 4
    q = np.zeros((1, 1, N, D), dtype=np.uint16)
    _, k, v = synth.qkv(1, 1, 1, N, D, seed=2)
    _, LSE = oracle.attention(q, k, v, Pattern(window=l, stride=s, n_global=G), 1.0)
    cnt = np.array([closed_row_count_strided(r, l, s, G) for r in range(N)])
    assert np.abs(LSE[0, 0] - np.log(cnt)).max() < 1e-12


def test_constant_values_give_constant_output():
    N, D = 260, 32
    q, k, _ = synth.qkv(1, 2, 1, N, D, seed=4)
    v = np.full((1, 1, N, D), 0x3F00, dtype=np.uint16)  # 0.5 in bf16
    O, _ = oracle.attention(q, k, v, Pattern(window=50, sinks=4), 1 / math.sqrt(D))
    assert np.abs(O - 0.5).max() < 1e-12


def test_empty_rows():
    N, D = 50, 8
    q, k, v = synth.qkv(1, 1, 1, N, D, seed=1)
    p = Pattern(window=-1)
    O, LSE = oracle.attention(q, k, v, p, 1.0)
    assert np.all(O == 0) and np.all(np.isneginf(LSE))
    counts, index, _ = oracle.block_mask(p, N, 16)
    assert counts.sum() == 0 and np.all(index == -1)


def test_row_subset_matches_full():
    N, D = 200, 16
    q, k, v = synth.qkv(2, 4, 2, N, D, seed=8)
    p = Pattern(window=30, sinks=2)
    O, LSE = oracle.attention(q, k, v, p, 0.25)
    rows = np.array([0, 7, 199, 100, 31])
    O2, LSE2 = oracle.attention(q, k, v, p, 0.25, rows=rows)
    assert np.array_equal(O[:, :, rows], O2) and np.array_equal(LSE[:, :, rows], LSE2)


# ----------------------------------------------------------------------------
# Input generator sanity: a known distribution, and slices agree with the whole.

def test_generator_statistics_and_determinism():
    a = synth.normal_bf16((1 << 20,), 0, 0)
    b = synth.normal_bf16((1 << 20,), 0, 0)
    assert np.array_equal(a, b)
    x = synth.bf16_bits_to_float(a).astype(np.float64)
    assert abs(x.mean()) < 5e-3 and abs(x.std() - 1) < 5e-3
    assert abs((np.abs(x) < 1).mean() - 0.6827) < 3e-3
    c = synth.normal_bf16((1 << 20,), 0, 1)
    assert not np.array_equal(a, c)


# ----------------------------------------------------------------------------
# The other reading of global rows ("global tokens attend to every position",
# without the causal conjunction): `global_rows_see_all`.  Pinned by closed
# forms, not by a restatement of the rule.

def closed_row_count_see_all(q, N, l, s, G):
    """|A(q)| when rows q < G see all N keys; other rows as closed_row_count_strided."""
    return N if q < G else closed_row_count_strided(q, l, s, G)


@pytest.mark.parametrize("N,l,s,G", [(16384, 128, 128, 16), (300, 10, 7, 5), (64, 3, 5, 9), (50, -1, 4, 50)])
def test_global_rows_see_all_pair_count_closed_form(N, l, s, G):
    p = Pattern(window=l, stride=s, n_global=G, global_rows_see_all=1)
    want = sum(closed_row_count_see_all(q, N, l, s, G) for q in range(N))
    assert oracle.count_pairs(p, N) == want
    # the two readings differ by the keys after each global row: sum_{q < G} (N - 1 - q)
    causal = oracle.count_pairs(Pattern(window=l, stride=s, n_global=G), N)
    g = min(G, N)
    assert want - causal == g * (N - 1) - g * (g - 1) // 2


def test_global_rows_see_all_strided_global_workload_count():
    # the strided + global workload (N = 16384, local 128, stride 128, 16 global
    # tokens) under this reading: 3 387 352 causal pairs plus 16 * 16383 - 120
    assert oracle.count_pairs(Pattern(window=128, stride=128, n_global=16, global_rows_see_all=1),
                              16384) == 3_387_352 + 16 * 16383 - 120


def test_global_rows_see_all_zero_query_gives_log_count_and_mean():
    # Q = 0: LSE = ln |A(q)| (ln N on a global row) and O = the mean of V over A(q)
    N, D, l, s, G = 240, 8, 12, 9, 5
    q = np.zeros((1, 2, N, D), dtype=np.uint16)
    _, k, v = synth.qkv(1, 2, 1, N, D, seed=31)
    O, LSE = oracle.attention(q, k, v, Pattern(window=l, stride=s, n_global=G, global_rows_see_all=1), 0.7)
    cnt = np.array([closed_row_count_see_all(r, N, l, s, G) for r in range(N)])
    assert np.abs(LSE - np.log(cnt)[None, None]).max() < 1e-12
    vf = synth.bf16_bits_to_float(v).astype(np.float64)
    for r in range(G):  # a global row averages every key of the sequence
        assert np.abs(O[:, :, r] - vf[:, :, :].mean(axis=2)).max() < 1e-12


def test_row_counts_match_closed_forms():
    # per-row brute force (the bench's CPU arms count their work with it) against the closed forms
    N, w, s = 700, 40, 4
    rows = np.array([0, 1, 39, 40, 41, 44, 45, 300, 699])
    got = oracle.row_counts(Pattern(window=w, sinks=s), N, rows)
    assert list(got) == [min(r, w) + 1 + min(s, max(0, r - w)) for r in rows]
    got = oracle.row_counts(Pattern(window=10, stride=7, n_global=3), 300, np.arange(300))
    assert list(got) == [closed_row_count_strided(r, 10, 7, 3) for r in range(300)]
    assert oracle.row_counts(Pattern(window=10, stride=7, n_global=3), 300, np.arange(300)).sum() == \
        oracle.count_pairs(Pattern(window=10, stride=7, n_global=3), 300)
