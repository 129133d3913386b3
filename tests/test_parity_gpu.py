"""GPU parity: the CUDA forward kernel, called through the C ABI, against the
fp64 CPU oracle on the same seeded inputs.

Bars (stated in the task's target): O within max-abs 2e-2 and LSE within
max-abs 1e-3 of fp64; rows with no allowed key must give O = 0, LSE = -inf
exactly.  Small shapes are compared element by element; the full-size
workloads on sampled query rows (every query tile is sampled, with its first
and last row) that the oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_build_b200 as sa
import oracle
import synth
from synth.workloads import WORKLOADS

pytestmark = pytest.mark.gpu

O_TOL = 2e-2
LSE_TOL = 1e-3


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def run_gpu(q, k, v, pattern: sa.Pattern, block: int, scale: float):
    N = q.shape[2]
    mask = sa.build_block_mask(pattern, N, block).to_device("cuda")
    O, LSE = sa.fwd(to_dev(q), to_dev(k), to_dev(v), mask, pattern, scale=scale)
    assert sa.check_device() == sa.SA_OK
    return O.float().cpu().numpy(), LSE.cpu().numpy()


def compare(O, LSE, Oref, LSEref):
    assert O.shape == Oref.shape and LSE.shape == LSEref.shape
    empty = np.isneginf(LSEref)
    assert np.array_equal(np.isneginf(LSE), empty)
    assert np.all(O[empty] == 0)
    assert np.isfinite(O).all()
    o_err = np.abs(O - Oref).max() if O.size else 0.0
    l_err = np.abs(LSE[~empty] - LSEref[~empty]).max() if (~empty).any() else 0.0
    assert o_err <= O_TOL, f"O max-abs {o_err}"
    assert l_err <= LSE_TOL, f"LSE max-abs {l_err}"
    return o_err, l_err


def opattern(p: sa.Pattern):
    return oracle.Pattern(window=p.window, sinks=p.sinks, stride=p.stride, n_global=p.n_global, causal=p.causal,
                          area=p.area, summary=p.summary)


SMALL = [
    # (B, Hq, Hkv, N, D, pattern, block)
    (1, 2, 2, 512, 64, sa.Pattern(window=128, sinks=4), 64),
    (1, 2, 2, 1000, 128, sa.Pattern(window=300, sinks=4), 128),          # ragged tail
    (2, 4, 2, 777, 64, sa.Pattern(window=100, sinks=3), 64),             # ragged, GQA, 64-wide tiles
    (1, 3, 1, 640, 128, sa.Pattern(window=640), 128),                    # dense causal
    (1, 2, 2, 1280, 128, sa.Pattern(window=128, stride=128, n_global=16), 128),
    (1, 2, 1, 900, 64, sa.Pattern(window=20, stride=37, n_global=5), 128),
    (1, 1, 1, 384, 128, sa.Pattern(window=0), 128),                      # diagonal only
    (1, 2, 2, 256, 64, sa.Pattern(window=-1, sinks=8), 64),              # sinks only
    (1, 1, 1, 100, 128, sa.Pattern(window=30, sinks=2), 128),            # one partial tile
    (1, 1, 1, 1, 64, sa.Pattern(window=5), 64),                          # N = 1
    (1, 2, 2, 300, 128, sa.Pattern(window=-1, stride=1), 128),           # stride 1 = dense
    (1, 2, 2, 1100, 128, sa.Pattern(window=257, sinks=130), 64),         # sinks wider than a tile
    (2, 3, 3, 700, 128, sa.Pattern(window=200, sinks=4), 128),           # odd head count: a one-slot unit
    (1, 4, 4, 1536, 128, sa.Pattern(window=1024, sinks=4), 128),         # head pairs, own K/V per slot
    (3, 1, 1, 900, 64, sa.Pattern(window=256, sinks=4), 64),             # one head, batched: q-tile pairs
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"B{c[0]}H{c[1]}/{c[2]}N{c[3]}D{c[4]}b{c[6]}-{c[5]}")
def test_small_full_parity_split_units(case):
    """Every unit split: each query tile's kv list walked as two halves by the
    two slots and merged at the end (the path of small problems and of a partial last round)."""
    B, Hq, Hkv, N, D, p, block = case
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=N + D + 1)
    scale = 1 / math.sqrt(D)
    sa.set_debug(sa.DEBUG_SPLIT_ALL)
    try:
        O, LSE = run_gpu(q, k, v, p, block, scale)
    finally:
        sa.set_debug(0)
    Oref, LSEref = oracle.attention(q, k, v, opattern(p), scale)
    compare(O, LSE, Oref, LSEref)


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"B{c[0]}H{c[1]}/{c[2]}N{c[3]}D{c[4]}b{c[6]}-{c[5]}")
def test_small_full_parity(case):
    B, Hq, Hkv, N, D, p, block = case
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=N + D)
    scale = 1 / math.sqrt(D)
    O, LSE = run_gpu(q, k, v, p, block, scale)
    Oref, LSEref = oracle.attention(q, k, v, opattern(p), scale)
    compare(O, LSE, Oref, LSEref)


def test_empty_rows_give_zero_and_neg_inf():
    # no rule admits any pair: every row is empty, no kv tile is live
    B, Hq, Hkv, N, D = 1, 2, 2, 300, 128
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=7)
    O, LSE = run_gpu(q, k, v, sa.Pattern(window=-1), 128, 0.1)
    assert np.all(O == 0) and np.all(np.isneginf(LSE))


def test_zero_query_lse_is_log_count():
    N, D, w, s = 1000, 128, 300, 4
    q = np.zeros((1, 1, N, D), dtype=np.uint16)
    _, k, v = synth.qkv(1, 1, 1, N, D, seed=1)
    _, LSE = run_gpu(q, k, v, sa.Pattern(window=w, sinks=s), 128, 0.1)
    cnt = np.array([min(r, w) + 1 + min(s, max(0, r - w)) for r in range(N)])
    assert np.abs(LSE[0, 0] - np.log(cnt)).max() <= LSE_TOL


def test_empty_problem_is_a_no_op():
    q = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16, device="cuda")
    mask = sa.build_block_mask(sa.Pattern(window=4), 0, 64).to_device("cuda")
    O, LSE = sa.fwd(q, q, q, mask, sa.Pattern(window=4))
    assert O.shape == (1, 2, 0, 64) and LSE.shape == (1, 2, 0)


def sample_rows(N: int, per_tile: int = 2, extra: int = 0, seed: int = 0) -> np.ndarray:
    rows = set()
    for t in range(0, N, 128):
        rows.add(t)
        rows.add(min(N, t + 128) - 1)
    rng = np.random.default_rng(seed)
    rows |= set(rng.integers(0, N, size=extra).tolist())
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workload_parity_sampled(name):
    w = WORKLOADS[name]
    q, k, v = synth.qkv(w.B, w.Hq, w.Hkv, w.N, w.D, seed=w.seed)
    p = sa.Pattern(**w.pattern_args())
    O, LSE = run_gpu(q, k, v, p, w.block, w.scale)
    rows = sample_rows(w.N, extra=64) if w.N > 4096 else np.arange(w.N)
    Oref, LSEref = oracle.attention(q, k, v, opattern(p), w.scale, rows=rows)
    compare(O[:, :, rows], LSE[:, :, rows], Oref, LSEref)


@pytest.mark.parametrize("block,D", [(128, 128), (64, 64)])
def test_largest_tile_count(block, D):
    """The most tiles per side the kernel takes (4096: its step lists hold 12-bit
    tile indices), with a ragged last tile: N = 4096 * block - 37.  Sampled
    rows (both ends of every query tile and 64 more) against the oracle."""
    N = 4096 * block - 37
    B, Hq, Hkv = 1, 2, 1
    p = sa.Pattern(window=300, sinks=4, n_global=2)
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=9)
    O, LSE = run_gpu(q, k, v, p, block, 1 / math.sqrt(D))
    rows = sample_rows(N, extra=64)
    Oref, LSEref = oracle.attention(q, k, v, opattern(p), 1 / math.sqrt(D), rows=rows)
    compare(O[:, :, rows], LSE[:, :, rows], Oref, LSEref)


def test_repeat_calls_are_deterministic():
    w = WORKLOADS["w1024_s4_n8192"]
    q, k, v = synth.qkv(1, 2, 2, 4096, 128, seed=3)
    p = sa.Pattern(**w.pattern_args())
    O1, L1 = run_gpu(q, k, v, p, 128, w.scale)
    O2, L2 = run_gpu(q, k, v, p, 128, w.scale)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


@pytest.mark.parametrize("B,Hq,Hkv,N,D,block,pinned", [
    (1, 4, 2, 1000, 128, 128, True),   # 2 chunks of one kv head
    (2, 6, 3, 777, 64, 64, True),      # 6 chunks across the batch, ragged, block 64
    (3, 4, 4, 384, 128, 128, True),    # 12 kv heads in 8 chunks of one or two
    (1, 2, 1, 640, 128, 128, False),   # pageable host memory, one chunk
])
def test_host_buffer_entry_point_matches_device_entry_point(B, Hq, Hkv, N, D, block, pinned):
    """The host-buffer call (chunks of kv heads, copies overlapping the kernels)
    gives the device call's output bit for bit, and both agree with the oracle.
    At these sizes the whole problem and every chunk have at most half as many
    work units as SMs, so both calls split every unit alike."""
    p = sa.Pattern(window=200, sinks=4)
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=21)
    O, LSE = run_gpu(q, k, v, p, block, 1 / math.sqrt(D))
    mask = sa.build_block_mask(p, N, block)
    host = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    pin = (lambda a: host(a).pin_memory()) if pinned else host
    Oh = torch.full((B, Hq, N, D), float("nan"), dtype=torch.bfloat16)
    Lh = torch.full((B, Hq, N), float("nan"), dtype=torch.float32)
    if pinned:
        Oh, Lh = Oh.pin_memory(), Lh.pin_memory()
    ws = torch.empty(sa.fwd_host_workspace_bytes(B, Hq, Hkv, N, D), dtype=torch.uint8, device="cuda")
    for _ in range(2):  # a second call on the same streams and workspace
        sa.fwd_host(pin(q), pin(k), pin(v), mask, p, Oh, Lh, ws)
        assert np.array_equal(Oh.float().numpy(), O) and np.array_equal(Lh.numpy(), LSE)
    Oref, Lref = oracle.attention(q, k, v, oracle.Pattern(window=200, sinks=4), 1 / math.sqrt(D))
    compare(Oh.float().numpy(), Lh.numpy(), Oref, Lref)


def test_host_buffer_async_calls_in_a_row():
    """Three queued host-buffer calls on different inputs, then one wait: each
    output equals the device call's on its inputs, bit for bit (the calls share
    the workspace; their copies overlap, the ordering keeps them apart).  The
    whole problem has more units than half the SMs and its chunks fewer, so
    the test hook splits every unit on both sides to give them one plan."""
    B, Hq, Hkv, N, D = 2, 8, 4, 1536, 128
    p = sa.Pattern(window=300, sinks=4)
    mask = sa.build_block_mask(p, N, 128)
    ws = torch.empty(sa.fwd_host_workspace_bytes(B, Hq, Hkv, N, D), dtype=torch.uint8, device="cuda")
    pin = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
    runs = []
    sa.set_debug(sa.DEBUG_SPLIT_ALL)
    try:
        for i in range(3):
            q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=40 + i)
            Oh = torch.empty((B, Hq, N, D), dtype=torch.bfloat16).pin_memory()
            Lh = torch.empty((B, Hq, N), dtype=torch.float32).pin_memory()
            ins = (pin(q), pin(k), pin(v))
            sa.fwd_host(*ins, mask, p, Oh, Lh, ws, wait=False)
            runs.append((q, k, v, ins, Oh, Lh))
        torch.cuda.synchronize()
        assert sa.check_device() == sa.SA_OK
        for q, k, v, _, Oh, Lh in runs:
            O, LSE = run_gpu(q, k, v, p, 128, 1 / math.sqrt(D))
            assert np.array_equal(Oh.float().numpy(), O) and np.array_equal(Lh.numpy(), LSE)
    finally:
        sa.set_debug(0)
    Oref, Lref = oracle.attention(q, k, v, oracle.Pattern(window=300, sinks=4), 1 / math.sqrt(D))
    compare(Oh.float().numpy(), Lh.numpy(), Oref, Lref)


def test_device_timeout_is_reported_and_context_survives():
    """The test hook skips the Q tile load, so the kernel's bounded waits
    expire (about 10 ms each); the status comes back as a timeout and the
    next ordinary call on the same context is correct."""
    B, Hq, Hkv, N, D = 1, 1, 1, 256, 128
    p = sa.Pattern(window=64, sinks=4)
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=5)
    mask = sa.build_block_mask(p, N, 128).to_device("cuda")
    try:
        sa.set_debug(sa.DEBUG_SKIP_Q_LOAD, 20_000_000)
        sa.fwd(to_dev(q), to_dev(k), to_dev(v), mask, p)
        assert sa.check_device() == sa.SA_ERR_DEVICE_TIMEOUT
    finally:
        sa.set_debug(0, 0)
    assert sa.check_device() == sa.SA_OK  # the word was cleared
    O, LSE = run_gpu(q, k, v, p, 128, 1 / math.sqrt(D))
    Oref, LSEref = oracle.attention(q, k, v, opattern(p), 1 / math.sqrt(D))
    compare(O, LSE, Oref, LSEref)


HEAD_CASES = [
    # (B, Hq, Hkv, N, D, block, patterns, pattern index per query head)
    (1, 4, 4, 1000, 128, 128,
     [sa.Pattern(window=200, sinks=4), sa.Pattern(window=64, stride=128, n_global=16), sa.Pattern(window=-1, sinks=8)],
     [0, 1, 2, 0]),
    # two query heads of one kv group under different patterns (their unit's step list is a union)
    (2, 4, 2, 777, 64, 64, [sa.Pattern(window=100, sinks=3), sa.Pattern(window=0, stride=37, n_global=5)], [0, 1, 1, 0]),
    (1, 6, 2, 1300, 128, 128,
     [sa.Pattern(window=300), sa.Pattern(window=1300), sa.Pattern(window=20, sinks=130)], [0, 1, 2, 2, 1, 0]),
    # one query head of each kv group sees no key at all: in every unit one slot has
    # no live step (its rows are O = 0, LSE = -inf) while the other runs
    (1, 4, 2, 900, 128, 128, [sa.Pattern(window=200, sinks=4), sa.Pattern(window=-1)], [0, 1, 1, 0]),
    (1, 4, 2, 700, 64, 64, [sa.Pattern(window=-1), sa.Pattern(window=90, sinks=2)], [0, 1, 1, 0]),
    # the most patterns the table holds (8), one per head of a batch of 16 heads on 4 kv heads,
    # causal and not, with stripes and summary columns
    (1, 16, 4, 1100, 64, 128,
     [sa.Pattern(window=100, sinks=4), sa.Pattern(window=40, stride=64, n_global=3), sa.Pattern(window=-1, sinks=20),
      sa.Pattern(window=1100), sa.Pattern(window=60, causal=0), sa.Pattern(window=-1, causal=0, area=275),
      sa.Pattern(window=-1, area=128, summary=16), sa.Pattern(window=0)],
     [0, 1, 2, 3, 4, 5, 6, 7, 7, 6, 5, 4, 3, 2, 1, 0]),
]


def run_heads(q, k, v, patterns, heads, block, scale):
    N = q.shape[2]
    masks = [sa.build_block_mask(p, N, block).to_device("cuda") for p in patterns]
    O, LSE = sa.fwd_heads(to_dev(q), to_dev(k), to_dev(v), masks, patterns, heads, scale=scale)
    assert sa.check_device() == sa.SA_OK
    return O.float().cpu().numpy(), LSE.cpu().numpy()


def oracle_heads(q, k, v, patterns, heads, scale):
    """Each query head by itself under its own pattern (heads are independent)."""
    Hq, Hkv = q.shape[1], k.shape[1]
    outs, lses = [], []
    for h in range(Hq):
        hk = h // (Hq // Hkv)
        O, L = oracle.attention(np.ascontiguousarray(q[:, h:h + 1]), np.ascontiguousarray(k[:, hk:hk + 1]),
                                np.ascontiguousarray(v[:, hk:hk + 1]), opattern(patterns[heads[h]]), scale)
        outs.append(O)
        lses.append(L)
    return np.concatenate(outs, axis=1), np.concatenate(lses, axis=1)


@pytest.mark.parametrize("split", [False, True], ids=["whole", "split"])
@pytest.mark.parametrize("case", HEAD_CASES, ids=lambda c: f"B{c[0]}H{c[1]}/{c[2]}N{c[3]}D{c[4]}b{c[5]}")
def test_per_head_patterns(case, split):
    B, Hq, Hkv, N, D, block, patterns, heads = case
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=N + 3)
    scale = 1 / math.sqrt(D)
    if split:
        sa.set_debug(sa.DEBUG_SPLIT_ALL)
    try:
        O, LSE = run_heads(q, k, v, patterns, heads, block, scale)
    finally:
        sa.set_debug(0)
    Oref, LSEref = oracle_heads(q, k, v, patterns, heads, scale)
    compare(O, LSE, Oref, LSEref)


def test_per_head_entry_with_one_pattern_equals_fwd():
    B, Hq, Hkv, N, D = 1, 4, 2, 1500, 128
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=11)
    p = sa.Pattern(window=256, sinks=4)
    scale = 1 / math.sqrt(D)
    O1, L1 = run_heads(q, k, v, [p], [0] * Hq, 128, scale)
    O2, L2 = run_gpu(q, k, v, p, 128, scale)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


GENERAL_CASES = [
    # (B, Hq, Hkv, N, D, pattern, block): without causality, and stripes
    (1, 2, 2, 1600, 64, sa.Pattern(window=-1, causal=0, area=400), 128),      # Area Attention, 4 x 400
    (2, 2, 1, 1000, 128, sa.Pattern(window=100, causal=0), 128),              # two-sided window, GQA
    (1, 2, 2, 700, 64, sa.Pattern(window=700, causal=0), 64),                 # dense, no causality
    (1, 3, 3, 900, 128, sa.Pattern(window=-1, sinks=4, n_global=3, causal=0, area=200), 128),
    (1, 2, 2, 1100, 64, sa.Pattern(window=20, causal=1, area=300), 64),       # block-causal stripes + band
    (1, 1, 1, 333, 128, sa.Pattern(window=10, causal=0, area=50), 128),       # ragged, stripes inside a tile
    (1, 2, 2, 2048, 128, sa.Pattern(window=-1, area=128, summary=16), 128),   # fixed pattern, blocks = tiles
    (2, 2, 1, 1000, 64, sa.Pattern(window=-1, area=100, summary=10), 64),     # fixed pattern, ragged blocks
    (1, 2, 2, 700, 128, sa.Pattern(window=-1, causal=0, area=24, summary=3), 128),  # short blocks, no causality
]


@pytest.mark.parametrize("split", [False, True], ids=["whole", "split"])
@pytest.mark.parametrize("case", GENERAL_CASES, ids=lambda c: f"B{c[0]}H{c[1]}/{c[2]}N{c[3]}D{c[4]}b{c[6]}-{c[5]}")
def test_general_pattern_parity(case, split):
    B, Hq, Hkv, N, D, p, block = case
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=N + 11)
    scale = 1 / math.sqrt(D)
    if split:
        sa.set_debug(sa.DEBUG_SPLIT_ALL)
    try:
        O, LSE = run_gpu(q, k, v, p, block, scale)
    finally:
        sa.set_debug(0)
    Oref, LSEref = oracle.attention(q, k, v, opattern(p), scale)
    compare(O, LSE, Oref, LSEref)


def test_per_head_mix_of_causal_and_area():
    B, Hq, Hkv, N, D, block = 1, 4, 2, 1600, 64, 128
    patterns = [sa.Pattern(window=256, sinks=4), sa.Pattern(window=-1, causal=0, area=400)]
    heads = [0, 1, 1, 0]
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=21)
    scale = 1 / math.sqrt(D)
    O, LSE = run_heads(q, k, v, patterns, heads, block, scale)
    Oref, LSEref = oracle_heads(q, k, v, patterns, heads, scale)
    compare(O, LSE, Oref, LSEref)


# ----------------------------------------------------------------------------
# Stride-aware path: pass 1 (pattern without its stride, token order), pass 2
# (the remaining stride pairs on tokens grouped by residue), merged; compared
# with the oracle under the whole pattern.

def run_stride(q, k, v, pattern: sa.Pattern, block: int, scale: float):
    N = q.shape[2]
    pass1, pass2 = sa.stride_plan(pattern, N, block)
    O, LSE = sa.fwd_stride(to_dev(q), to_dev(k), to_dev(v), pass1.to_device("cuda"), pass2.to_device("cuda"),
                           pattern, scale=scale)
    assert sa.check_device() == sa.SA_OK
    return O.float().cpu().numpy(), LSE.cpu().numpy()


STRIDE_CASES = [
    # (B, Hq, Hkv, N, D, pattern, block)
    (1, 2, 2, 2048, 128, sa.Pattern(window=128, stride=128, n_global=16), 128),  # groups of 16 tokens
    (2, 4, 2, 1024, 64, sa.Pattern(window=100, stride=4, sinks=3), 64),          # GQA, groups of 256
    (1, 2, 2, 1536, 128, sa.Pattern(window=-1, stride=12), 128),                 # stride only, groups of 128
    (1, 2, 1, 4096, 128, sa.Pattern(window=256, stride=32, n_global=40), 128),   # global wider than the stride
    (1, 1, 1, 640, 64, sa.Pattern(window=3, stride=5, sinks=1), 128),            # groups straddle tiles
]


@pytest.mark.parametrize("split", [False, True], ids=["whole", "split"])
@pytest.mark.parametrize("case", STRIDE_CASES, ids=lambda c: f"B{c[0]}H{c[1]}/{c[2]}N{c[3]}D{c[4]}b{c[6]}-{c[5]}")
def test_stride_aware_parity(case, split):
    B, Hq, Hkv, N, D, p, block = case
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=N + 3)
    scale = 1 / math.sqrt(D)
    if split:
        sa.set_debug(sa.DEBUG_SPLIT_ALL)
    try:
        O, LSE = run_stride(q, k, v, p, block, scale)
    finally:
        sa.set_debug(0)
    Oref, LSEref = oracle.attention(q, k, v, opattern(p), scale)
    compare(O, LSE, Oref, LSEref)


def test_stride_aware_workload_sampled():
    w = WORKLOADS["strided_global_n16384"]
    q, k, v = synth.qkv(w.B, w.Hq, w.Hkv, w.N, w.D, seed=w.seed)
    p = sa.Pattern(**w.pattern_args())
    O, LSE = run_stride(q, k, v, p, w.block, w.scale)
    rows = sample_rows(w.N, extra=64)
    Oref, LSEref = oracle.attention(q, k, v, opattern(p), w.scale, rows=rows)
    compare(O[:, :, rows], LSE[:, :, rows], Oref, LSEref)
    # and the plain path on the same inputs agrees within the bars
    O2, LSE2 = run_gpu(q, k, v, p, w.block, w.scale)
    assert np.abs(O - O2).max() <= O_TOL and np.abs(LSE - LSE2).max() <= LSE_TOL


def test_mask_the_device_cannot_read_is_refused():
    """Through the C ABI: a mask in pageable host memory is refused with
    SA_ERR_INVALID_ARG before any launch (forward and backward); one in pinned
    host memory, which the device reads over the bus, gives the device mask's
    output bit for bit."""
    import ctypes
    B, Hq, Hkv, N, D = 1, 2, 1, 600, 64
    p = sa.Pattern(window=150, sinks=4)
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=77)
    Q, K, V = to_dev(q), to_dev(k), to_dev(v)
    hmask = sa.build_block_mask(p, N, 128)
    O_ref, L_ref = sa.fwd(Q, K, V, hmask.to_device("cuda"), p)
    torch.cuda.synchronize()

    def c_fwd(mask, O, L):
        return sa.lib.sparse_attn_fwd(Q.data_ptr(), K.data_ptr(), V.data_ptr(), ctypes.byref(mask._c()),
                                      ctypes.byref(p._c()), ctypes.byref(sa._Shape(B, Hq, Hkv, N, D)),
                                      1 / math.sqrt(D), O.data_ptr(), L.data_ptr(), None)

    O = torch.full_like(O_ref, float("nan"))
    L = torch.full_like(L_ref, float("nan"))
    assert c_fwd(hmask, O, L) == sa.SA_ERR_INVALID_ARG  # numpy: pageable host memory
    torch.cuda.synchronize()
    assert torch.isnan(O.float()).all() and torch.isnan(L).all()  # nothing ran
    pinned = sa.BlockMask(*(torch.from_numpy(a).pin_memory() for a in (hmask.counts, hmask.index, hmask.full)),
                          hmask.block, hmask.n_live, hmask.n_full, hmask.max_per_row, N)
    assert c_fwd(pinned, O, L) == sa.SA_OK
    torch.cuda.synchronize()
    assert sa.check_device() == sa.SA_OK
    assert torch.equal(O, O_ref) and torch.equal(L, L_ref)

    ht = sa.transpose_block_mask(hmask)
    g = [torch.empty_like(t) for t in (Q, K, V)]
    ws = torch.empty(sa.bwd_workspace_bytes(B, Hq, Hkv, N, D), dtype=torch.uint8, device="cuda")
    rc = sa.lib.sparse_attn_bwd(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O_ref.data_ptr(), L_ref.data_ptr(),
                                Q.data_ptr(), ctypes.byref(ht._c()), ctypes.byref(p._c()),
                                ctypes.byref(sa._Shape(B, Hq, Hkv, N, D)), 1 / math.sqrt(D), g[0].data_ptr(),
                                g[1].data_ptr(), g[2].data_ptr(), ws.data_ptr(), ws.numel(), None)
    assert rc == sa.SA_ERR_INVALID_ARG


def test_host_buffer_entry_point_at_the_headline_size():
    """The host-buffer path on the full headline workload (16 heads cut into
    chunks of 8, 4, 2, 1, 1): sampled rows against the oracle, and the whole
    output against the device call within rounding (the chunks are smaller
    problems than the whole, so their work plans may split units differently)."""
    w = WORKLOADS["w1024_s4_n8192"]
    q, k, v = synth.qkv(w.B, w.Hq, w.Hkv, w.N, w.D, seed=w.seed)
    p = sa.Pattern(**w.pattern_args())
    O, LSE = run_gpu(q, k, v, p, w.block, w.scale)
    pin = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
    Oh = torch.empty((w.B, w.Hq, w.N, w.D), dtype=torch.bfloat16).pin_memory()
    Lh = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32).pin_memory()
    ws = torch.empty(sa.fwd_host_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.D), dtype=torch.uint8, device="cuda")
    sa.fwd_host(pin(q), pin(k), pin(v), sa.build_block_mask(p, w.N, w.block), p, Oh, Lh, ws, scale=w.scale)
    Oh, Lh = Oh.float().numpy(), Lh.numpy()
    assert np.abs(Oh - O).max() <= 1e-2 and np.abs(Lh - LSE).max() <= 1e-4
    rows = sample_rows(w.N, extra=64)
    Oref, LSEref = oracle.attention(q, k, v, opattern(p), w.scale, rows=rows)
    compare(Oh[:, :, rows], Lh[:, :, rows], Oref, LSEref)
