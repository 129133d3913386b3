"""Seeded random shapes and patterns through the forward and backward kernels
(C ABI) against the fp64 oracle, every row: batch 1-2, 1-3 kv heads with
groups of 1, 2 or 4 query heads, N from 1 to 2500 (ragged tails), D 64 or
128, tiles of 64 or 128, and random mixes of the pattern's rules (band,
sinks, stride, global tokens, no causality, stripes, summary columns), some
of which leave rows without any key.  Half of the forward cases split every
work unit.  Bars as in the other parity tests."""
import math

import numpy as np
import pytest

import block_sparse_attention_build_b200 as sa
import oracle
import synth

from test_parity_gpu import compare, opattern, run_gpu
from test_parity_bwd_gpu import compare_grads, inputs, run_gpu_bwd

pytestmark = pytest.mark.gpu


def random_pattern(rng, N):
    causal = int(rng.random() < 0.75)
    window = int(rng.integers(-1, max(1, N // 2))) if rng.random() < 0.8 else -1
    sinks = int(rng.integers(0, 200)) if rng.random() < 0.4 else 0
    stride = int(rng.integers(1, 300)) if causal and rng.random() < 0.3 else 0
    n_global = int(rng.integers(0, 50)) if rng.random() < 0.3 else 0
    area = summary = 0
    if stride == 0 and rng.random() < 0.25:
        area = int(rng.integers(16, 800))
        summary = int(rng.integers(1, area + 1)) if rng.random() < 0.5 else 0
    return sa.Pattern(window=window, sinks=sinks, stride=stride, n_global=n_global, causal=causal, area=area,
                      summary=summary)


def random_case(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 3))
    Hkv = int(rng.integers(1, 4))
    group = int(rng.choice([1, 2, 4]))
    N = int(rng.integers(1, 2501))
    D = int(rng.choice([64, 128]))
    block = int(rng.choice([64, 128]))
    return B, Hkv * group, Hkv, N, D, block, random_pattern(rng, N)


FWD_SEEDS = list(range(1000, 1030))
BWD_SEEDS = list(range(2000, 2012))


@pytest.mark.parametrize("seed", FWD_SEEDS)
def test_random_forward_parity(seed):
    B, Hq, Hkv, N, D, block, p = random_case(seed)
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=seed)
    scale = 1 / math.sqrt(D)
    split = seed % 2 == 1
    try:
        sa.set_debug(sa.DEBUG_SPLIT_ALL if split else 0, 0)
        O, LSE = run_gpu(q, k, v, p, block, scale)
    finally:
        sa.set_debug(0, 0)
    Oref, LSEref = oracle.attention(q, k, v, opattern(p), scale)
    compare(O, LSE, Oref, LSEref)


@pytest.mark.parametrize("seed", BWD_SEEDS)
def test_random_backward_parity(seed):
    B, Hq, Hkv, N, D, _, p = random_case(seed)
    q, k, v, do = inputs(B, Hq, Hkv, N, D, seed=seed)
    scale = 1 / math.sqrt(D)
    got = run_gpu_bwd(q, k, v, do, p, scale)
    _, _, dQ, dK, dV = oracle.attention_bwd(q, k, v, do, opattern(p), scale)
    compare_grads(got, (dQ, dK, dV))
