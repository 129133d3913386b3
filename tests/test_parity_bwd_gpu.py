"""GPU parity of the backward pass: dQ, dK, dV from the CUDA kernels (called
through the C ABI, fed by the CUDA forward's O and LSE) against the fp64
oracle's gradients of the masked attention on the same seeded inputs.

Bar: per tensor, max |GPU - oracle| <= GRAD_TOL * max(max |oracle|, FLOOR).
The bf16 rounding of P and dS inside the kernel and of O, dQ, dK, dV at the
boundary are each 2^-9 relative; GRAD_TOL leaves headroom over their sum.
FLOOR covers gradients that cancel exactly (a query that sees only itself has
O = V, so dP - Delta = 0 and dQ = 0): fp32 sums of terms of size |dO||V| leave
a residue near 2^-24 * D * |dO||V|, about 1e-6 here, well under
GRAD_TOL * FLOOR = 2e-5.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_build_b200 as sa
import oracle
import synth

pytestmark = pytest.mark.gpu

GRAD_TOL = 2e-2
FLOOR = 1e-3


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def opattern(p: sa.Pattern):
    return oracle.Pattern(window=p.window, sinks=p.sinks, stride=p.stride, n_global=p.n_global, causal=p.causal,
                          area=p.area, summary=p.summary)


def inputs(B, Hq, Hkv, N, D, seed):
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=seed)
    do = synth.qkv(B, Hq, Hkv, N, D, seed=seed + 7919)[0]
    return q, k, v, do


def run_gpu_bwd(q, k, v, do, p: sa.Pattern, scale: float):
    N = q.shape[2]
    mask = sa.build_block_mask(p, N, 128)
    dmask = mask.to_device("cuda")
    dmask_t = sa.transpose_block_mask(mask).to_device("cuda")
    tq, tk, tv, tdo = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    O, LSE = sa.fwd(tq, tk, tv, dmask, p, scale=scale)
    dq, dk, dv = sa.bwd(tq, tk, tv, O, LSE, tdo, dmask_t, p, scale=scale)
    assert sa.check_device() == sa.SA_OK
    return [t.float().cpu().numpy() for t in (dq, dk, dv)]


def compare_grads(got, ref):
    """Asserts the bar; returns the relative errors (for the record)."""
    rel = []
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        assert g.shape == r.shape, name
        assert np.isfinite(g).all(), name
        scale = np.abs(r).max()
        err = np.abs(g - r).max()
        assert err <= GRAD_TOL * max(scale, FLOOR), f"{name}: max err {err} vs max |ref| {scale}"
        rel.append(err / max(scale, FLOOR))
    print("relative errors dQ dK dV:", " ".join(f"{x:.2e}" for x in rel))
    return rel


CASES = [
    # (B, Hq, Hkv, N, D, pattern)
    (1, 2, 2, 512, 64, sa.Pattern(window=128, sinks=4)),               # the tiny workload (its forward tiles are 64)
    (1, 2, 2, 512, 128, sa.Pattern(window=128, sinks=4)),
    (1, 2, 2, 1000, 128, sa.Pattern(window=300, sinks=4)),             # ragged tail
    (2, 4, 2, 777, 64, sa.Pattern(window=100, sinks=3)),               # GQA, D = 64, ragged
    (1, 3, 1, 640, 128, sa.Pattern(window=640)),                       # dense causal, group of 3
    (1, 2, 2, 1280, 128, sa.Pattern(window=128, stride=128, n_global=16)),
    (1, 2, 1, 900, 64, sa.Pattern(window=20, stride=37, n_global=5)),  # odd stride: partial tiles everywhere
    (1, 1, 1, 384, 128, sa.Pattern(window=0)),                         # diagonal only
    (1, 2, 2, 256, 64, sa.Pattern(window=-1, sinks=8)),                # sinks only
    (1, 1, 1, 100, 128, sa.Pattern(window=30, sinks=2)),               # one partial tile
    (1, 1, 1, 1, 64, sa.Pattern(window=5)),                            # N = 1
    (1, 2, 2, 1100, 128, sa.Pattern(window=257, sinks=130)),           # sinks wider than a tile
    (1, 2, 2, 1600, 64, sa.Pattern(window=-1, causal=0, area=400)),    # Area Attention, 4 x 400
    (2, 2, 1, 1000, 128, sa.Pattern(window=100, causal=0)),            # two-sided window, GQA
    (1, 2, 2, 900, 128, sa.Pattern(window=-1, sinks=4, n_global=3, causal=0, area=200)),
    (1, 2, 2, 1100, 64, sa.Pattern(window=20, causal=1, area=300)),    # block-causal stripes + band
    (1, 2, 2, 2048, 128, sa.Pattern(window=-1, area=128, summary=16)),  # fixed pattern
    (1, 2, 1, 1000, 64, sa.Pattern(window=-1, causal=0, area=24, summary=3)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}H{c[1]}/{c[2]}N{c[3]}D{c[4]}-{c[5]}")
def test_bwd_full_parity(case):
    B, Hq, Hkv, N, D, p = case
    q, k, v, do = inputs(B, Hq, Hkv, N, D, seed=N + D + 5)
    scale = 1 / math.sqrt(D)
    got = run_gpu_bwd(q, k, v, do, p, scale)
    _, _, dQ, dK, dV = oracle.attention_bwd(q, k, v, do, opattern(p), scale)
    compare_grads(got, (dQ, dK, dV))


def test_bwd_no_allowed_pair_gives_zero_gradients():
    q, k, v, do = inputs(1, 2, 2, 300, 128, seed=3)
    dq, dk, dv = run_gpu_bwd(q, k, v, do, sa.Pattern(window=-1), 0.1)
    assert np.all(dq == 0) and np.all(dk == 0) and np.all(dv == 0)


def test_bwd_is_deterministic_up_to_dq_order():
    # dK and dV are accumulated in tensor memory in a fixed order: bit-identical
    # across runs; dQ sums tiles with global reductions whose order may vary
    q, k, v, do = inputs(1, 2, 2, 1000, 128, seed=4)
    p = sa.Pattern(window=300, sinks=4)
    a = run_gpu_bwd(q, k, v, do, p, 0.088)
    b = run_gpu_bwd(q, k, v, do, p, 0.088)
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])
    assert np.abs(a[0] - b[0]).max() <= 1e-2 * np.abs(a[0]).max()


def test_bwd_headline_size_two_heads():
    """The 8192-token window + sinks workload (16 heads) through the kernels;
    two heads checked against the oracle in full."""
    B, H, N, D = 1, 16, 8192, 128
    p = sa.Pattern(window=1024, sinks=4)
    q, k, v, do = inputs(B, H, H, N, D, seed=0)
    scale = 1 / math.sqrt(D)
    dq, dk, dv = run_gpu_bwd(q, k, v, do, p, scale)
    for h in (0, 11):
        sl = slice(h, h + 1)
        _, _, rq, rk, rv = oracle.attention_bwd(q[:, sl], k[:, sl], v[:, sl], do[:, sl], opattern(p), scale)
        compare_grads((dq[:, sl], dk[:, sl], dv[:, sl]), (rq, rk, rv))


SPLIT_CASES = [
    # lists longer than 32 steps, walked as several work items whose dK, dV
    # add up in fp32 sums (forced by the test hook)
    (1, 4, 2, 4096, 128, sa.Pattern(window=512, sinks=4)),    # the sink tile: 32 query tiles x 2 heads
    (1, 2, 1, 4608, 64, sa.Pattern(window=4608)),             # dense causal: up to 36 x 2 steps per tile
    (2, 8, 1, 1280, 128, sa.Pattern(window=256, sinks=8)),    # a group of 8 heads: 8 steps per query tile
    (1, 2, 2, 4100, 128, sa.Pattern(window=-1, sinks=130, n_global=3)),  # two sink tiles, ragged tail
]


@pytest.mark.parametrize("case", SPLIT_CASES, ids=lambda c: f"B{c[0]}H{c[1]}/{c[2]}N{c[3]}D{c[4]}-{c[5]}")
def test_bwd_split_items_parity(case):
    B, Hq, Hkv, N, D, p = case
    q, k, v, do = inputs(B, Hq, Hkv, N, D, seed=N + D + 17)
    scale = 1 / math.sqrt(D)
    mask_t = sa.transpose_block_mask(sa.build_block_mask(p, N, 128))
    assert mask_t.counts.max() * (Hq // Hkv) > 32  # some list is long enough to split
    try:
        sa.set_debug(sa.DEBUG_BWD_SPLIT, 0)
        got = run_gpu_bwd(q, k, v, do, p, scale)
    finally:
        sa.set_debug(0, 0)
    _, _, dQ, dK, dV = oracle.attention_bwd(q, k, v, do, opattern(p), scale)
    compare_grads(got, (dQ, dK, dV))


def test_bwd_narrow_window_many_heads_full_size_two_kv_heads():
    """The 16 384-token narrow-window workload with 64 query heads on 8 kv heads,
    at full size: every query tile attends to the sink tile, so kv tile 0's list
    (128 query tiles x 8 heads) is split across work items without any test
    hook.  Two kv heads (their 16 query heads) are checked against the oracle."""
    B, Hq, Hkv, N, D = 2, 64, 8, 16384, 64
    p = sa.Pattern(window=128, sinks=4)
    q, k, v, do = inputs(B, Hq, Hkv, N, D, seed=0)
    scale = 1 / math.sqrt(D)
    dq, dk, dv = run_gpu_bwd(q, k, v, do, p, scale)
    group = Hq // Hkv
    for b, hk in ((0, 0), (1, 5)):
        sq, sk = slice(hk * group, (hk + 1) * group), slice(hk, hk + 1)
        _, _, rq, rk, rv = oracle.attention_bwd(q[b:b + 1, sq], k[b:b + 1, sk], v[b:b + 1, sk], do[b:b + 1, sq],
                                                opattern(p), scale)
        compare_grads((dq[b:b + 1, sq], dk[b:b + 1, sk], dv[b:b + 1, sk]), (rq, rk, rv))


HEAD_CASES = [
    # (B, Hq, Hkv, N, D, patterns, pattern of each query head)
    (1, 4, 2, 1000, 128, [sa.Pattern(window=200, sinks=4), sa.Pattern(window=64, stride=128, n_global=16)],
     [0, 1, 1, 0]),  # the two heads of each kv group differ
    (2, 4, 4, 777, 64, [sa.Pattern(window=100, sinks=3), sa.Pattern(window=-1, causal=0, area=200),
                        sa.Pattern(window=-1, area=128, summary=16)], [0, 1, 2, 1]),
]


def test_bwd_per_head_patterns():
    for B, Hq, Hkv, N, D, patterns, heads in HEAD_CASES:
        q, k, v, do = inputs(B, Hq, Hkv, N, D, seed=N + 13)
        scale = 1 / math.sqrt(D)
        masks = [sa.build_block_mask(p, N, 128) for p in patterns]
        dmasks = [m.to_device("cuda") for m in masks]
        dmasks_t = [sa.transpose_block_mask(m).to_device("cuda") for m in masks]
        tq, tk, tv, tdo = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
        O, LSE = sa.fwd_heads(tq, tk, tv, dmasks, patterns, heads, scale=scale)
        dq, dk, dv = sa.bwd_heads(tq, tk, tv, O, LSE, tdo, dmasks_t, patterns, heads, scale=scale)
        assert sa.check_device() == sa.SA_OK
        got = [t.float().cpu().numpy() for t in (dq, dk, dv)]
        # the oracle head by head; dK, dV of a kv head sum its query heads
        group = Hq // Hkv
        rq = np.zeros(q.shape)
        rk = np.zeros(k.shape)
        rv = np.zeros(v.shape)
        for h in range(Hq):
            hk = h // group
            sl, sk = slice(h, h + 1), slice(hk, hk + 1)
            _, _, a, b_, c_ = oracle.attention_bwd(q[:, sl], k[:, sk], v[:, sk], do[:, sl],
                                                   opattern(patterns[heads[h]]), scale)
            rq[:, sl] = a
            rk[:, sk] += b_
            rv[:, sk] += c_
        compare_grads(got, (rq, rk, rv))


def test_bwd_heads_with_one_pattern_equals_bwd():
    B, Hq, Hkv, N, D = 1, 4, 2, 1000, 128
    p = sa.Pattern(window=300, sinks=4)
    q, k, v, do = inputs(B, Hq, Hkv, N, D, seed=77)
    m = sa.build_block_mask(p, N, 128)
    mt = sa.transpose_block_mask(m).to_device("cuda")
    tq, tk, tv, tdo = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    O, LSE = sa.fwd(tq, tk, tv, m.to_device("cuda"), p)
    a = sa.bwd(tq, tk, tv, O, LSE, tdo, mt, p)
    b = sa.bwd_heads(tq, tk, tv, O, LSE, tdo, [mt], [p], [0] * Hq)
    torch.cuda.synchronize()
    # dK, dV are accumulated in a fixed order (bit-identical); dQ sums tiles with reductions
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert (a[0].float() - b[0].float()).abs().max().item() <= 1e-2 * a[0].float().abs().max().item()
