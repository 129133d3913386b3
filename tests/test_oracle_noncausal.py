"""Pins for the oracle's patterns without causality: the two-sided sliding
window ("Sparse-трансформеры" page, section "Основные шаблоны разреженности":
w neighbours on the left and on the right) and Area Attention ("Sparse
Attention" glossary page, section "Anwendungen": stripes of consecutive
tokens, attention only inside each stripe).  Each is checked against the
printed pair count, closed forms, a brute-force restatement of the rules on
tiny inputs, torch's scaled_dot_product_attention in fp64, the Q = 0
identity, and finite differences for the backward."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import Pattern
from test_oracle import read_golden, to_f64
from test_oracle_bwd import fd_pin_holds, torch_grads


def nc_sets(N, q, p: Pattern):
    """Allowed keys of query q, the rules of the pages as sets (no causality
    unless p.causal)."""
    s = set()
    if p.window >= 0:
        s |= set(range(max(0, q - p.window), min(N, q + p.window + 1)))
    s |= set(range(0, min(p.sinks, N)))
    s |= set(range(0, min(p.n_global, N)))
    if q < p.n_global:
        s |= set(range(N))
    if p.area > 0:
        a0 = (q // p.area) * p.area
        s |= set(range(a0, min(N, a0 + p.area)))
    if p.causal:
        s &= set(range(0, q + 1))
    return s


def test_printed_area_attention_pairs():
    g = read_golden("area_attention_pairs.txt")
    n, stripes, per = int(g["tokens"]), int(g["stripes"]), int(g["stripe_tokens"])
    assert stripes * per == n and n * n == int(g["full_pairs"])
    p = Pattern(window=-1, causal=0, area=per)
    pairs = oracle.count_pairs(p, n)
    assert pairs == float(g["evaluated_fraction"]) * int(g["full_pairs"]) == 640000


@pytest.mark.parametrize("N,w", [(1000, 37), (300, 0), (129, 200), (4096, 511)])
def test_two_sided_window_pair_count(N, w):
    p = Pattern(window=w, causal=0)
    closed = sum(min(q, w) + min(N - 1 - q, w) + 1 for q in range(N))
    assert oracle.count_pairs(p, N) == closed


@pytest.mark.parametrize("N,A", [(1600, 400), (1000, 128), (777, 100)])
def test_causal_area_pair_count(N, A):
    # block-causal: query q sees its stripe up to itself, q - A floor(q / A) + 1 keys
    p = Pattern(window=-1, causal=1, area=A)
    assert oracle.count_pairs(p, N) == sum(q - (q // A) * A + 1 for q in range(N))


TINY = [
    (Pattern(window=3, causal=0), 30, 8),
    (Pattern(window=-1, causal=0, area=10), 37, 8),
    (Pattern(window=2, sinks=3, causal=0, area=7), 33, 4),
    (Pattern(window=1, n_global=4, causal=0), 29, 8),
    (Pattern(window=-1, causal=1, area=6), 31, 8),
    (Pattern(window=40, causal=0), 25, 8),
]


@pytest.mark.parametrize("p,N,b", TINY)
def test_noncausal_block_mask_brute_force_tiny(p, N, b):
    sets = [nc_sets(N, q, p) for q in range(N)]
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
        assert list(index[i, : counts[i]]) == row_j and list(full[i, : counts[i]]) == row_f
    assert oracle.count_pairs(p, N) == sum(len(s) for s in sets)


def test_strided_without_causality_is_undefined():
    with pytest.raises(ValueError):
        oracle.allowed(Pattern(window=2, stride=4, causal=0), 5, 1)


def test_dense_noncausal_equals_sdpa():
    B, Hq, Hkv, N, D = 2, 4, 2, 90, 16
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=17)
    scale = 1 / math.sqrt(D)
    O, LSE = oracle.attention(q, k, v, Pattern(window=N, causal=0), scale)
    kt = to_f64(k).repeat_interleave(2, dim=1)
    vt = to_f64(v).repeat_interleave(2, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(to_f64(q), kt, vt, is_causal=False, scale=scale)
    assert np.abs(O - ref.numpy()).max() < 1e-12
    assert np.abs(LSE - torch.logsumexp(to_f64(q) @ kt.transpose(-1, -2) * scale, dim=-1).numpy()).max() < 1e-12


@pytest.mark.parametrize("p,N", [(Pattern(window=5, causal=0), 60), (Pattern(window=-1, causal=0, area=16), 70),
                                 (Pattern(window=2, sinks=2, n_global=3, causal=0, area=9), 50),
                                 (Pattern(window=-1, causal=1, area=12), 40)])
def test_noncausal_equals_sdpa_with_explicit_mask(p, N):
    B, Hq, Hkv, D = 1, 2, 1, 8
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=N)
    scale = 0.41
    O, LSE = oracle.attention(q, k, v, p, scale)
    mask = torch.zeros(N, N, dtype=torch.bool)
    for qi in range(N):
        mask[qi, sorted(nc_sets(N, qi, p))] = True
    kt, vt = to_f64(k).repeat_interleave(2, 1), to_f64(v).repeat_interleave(2, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(to_f64(q), kt, vt, attn_mask=mask, scale=scale)
    assert np.abs(O - ref.numpy()).max() < 1e-12


def test_zero_query_area_lse_is_log_stripe():
    # Q = 0: uniform weights over the stripe, LSE = ln 400 for every query of the printed example
    N, D, A = 1600, 8, 400
    q = np.zeros((1, 1, N, D), dtype=np.uint16)
    _, k, v = synth.qkv(1, 1, 1, N, D, seed=2)
    O, LSE = oracle.attention(q, k, v, Pattern(window=-1, causal=0, area=A), 0.5)
    assert np.abs(LSE - math.log(A)).max() < 1e-12
    vf = synth.bf16_bits_to_float(v).astype(np.float64)[0, 0]
    stripe_mean = vf.reshape(N // A, A, D).mean(axis=1).repeat(A, axis=0)
    assert np.abs(O[0, 0] - stripe_mean).max() < 1e-12


@pytest.mark.parametrize("case", [(1, 2, 1, 10, 3, Pattern(window=2, causal=0)),
                                  (1, 1, 1, 11, 2, Pattern(window=-1, sinks=1, causal=0, area=4))])
def test_noncausal_gradients_match_finite_differences(case):
    assert fd_pin_holds(oracle.default(), case)


def test_noncausal_gradients_equal_autograd():
    B, Hq, Hkv, N, D = 1, 2, 1, 48, 8
    p = Pattern(window=3, causal=0, area=16)
    q, k, v = (synth.bf16_bits_to_float(a).astype(np.float64) for a in synth.qkv(B, Hq, Hkv, N, D, seed=8))
    do = np.random.default_rng(3).standard_normal((B, Hq, N, D))
    mask = np.zeros((N, N), dtype=bool)
    for qi in range(N):
        mask[qi, sorted(nc_sets(N, qi, p))] = True
    O, _, dQ, dK, dV = oracle.attention_bwd(q, k, v, do, p, 0.3)
    rO, rq, rk, rv = torch_grads(q, k, v, do, 0.3, mask=mask)
    for a, b in ((O, rO), (dQ, rq), (dK, rk), (dV, rv)):
        assert np.abs(a - b).max() <= 1e-10


# ----------------------------------------------------------------------------
# The "fixed" pattern ("Sparse-трансформеры" page, section "Основные шаблоны
# разреженности"): local attention inside blocks of `area` tokens, plus the
# last `summary` positions of every block as keys for all later queries.

def fixed_sets(N, q, A, c, causal=1):
    s = set(range((q // A) * A, min(N, (q // A) * A + A)))
    s |= {kv for kv in range(N) if kv % A >= A - c}
    if causal:
        s &= set(range(q + 1))
    return s


@pytest.mark.parametrize("N,A,c", [(1024, 128, 16), (1000, 100, 10), (333, 64, 1), (257, 32, 32)])
def test_fixed_pattern_pair_count_closed_form(N, A, c):
    # causal: q mod A + 1 keys of its own block, plus c summary keys in each earlier block
    p = Pattern(window=-1, causal=1, area=A, summary=c)
    closed = sum(q % A + 1 + (q // A) * min(c, A) for q in range(N))
    if c >= A:
        closed = N * (N + 1) // 2  # every key is a summary key: dense causal
    assert oracle.count_pairs(p, N) == closed


@pytest.mark.parametrize("p,N", [(Pattern(window=-1, causal=1, area=8, summary=2), 37),
                                 (Pattern(window=1, causal=0, area=6, summary=1), 29),
                                 (Pattern(window=-1, sinks=2, causal=1, area=10, summary=3), 41)])
def test_fixed_pattern_brute_force_and_sdpa(p, N):
    def sets(q):
        s = fixed_sets(N, q, p.area, p.summary, p.causal) | nc_sets(N, q, Pattern(
            window=p.window, sinks=p.sinks, n_global=p.n_global, causal=p.causal, area=p.area))
        return s
    for q in range(N):
        for kv in range(N):
            assert oracle.allowed(p, q, kv) == (kv in sets(q))
    B, Hq, Hkv, D = 1, 2, 1, 8
    qq, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=N + 1)
    O, _ = oracle.attention(qq, k, v, p, 0.4)
    mask = torch.zeros(N, N, dtype=torch.bool)
    for qi in range(N):
        mask[qi, sorted(sets(qi))] = True
    kt, vt = to_f64(k).repeat_interleave(2, 1), to_f64(v).repeat_interleave(2, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(to_f64(qq), kt, vt, attn_mask=mask, scale=0.4)
    assert np.abs(O - ref.numpy()).max() < 1e-12


def test_fixed_pattern_zero_query_lse():
    N, D, A, c = 1024, 8, 128, 16
    q = np.zeros((1, 1, N, D), dtype=np.uint16)
    _, k, v = synth.qkv(1, 1, 1, N, D, seed=3)
    _, LSE = oracle.attention(q, k, v, Pattern(window=-1, causal=1, area=A, summary=c), 0.5)
    cnt = np.array([r % A + 1 + (r // A) * c for r in range(N)])
    assert np.abs(LSE[0, 0] - np.log(cnt)).max() < 1e-12


def test_fixed_pattern_gradients_match_finite_differences():
    assert fd_pin_holds(oracle.default(), (1, 1, 1, 12, 2, Pattern(window=-1, causal=1, area=4, summary=1)))
