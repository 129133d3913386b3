"""Pins of the backward oracle (gradients of the masked attention of the
"Sparse-трансформеры" page, section "Как это выглядит в коде", with respect to
Q, K, V).  None of them retypes the oracle's formulas: each checks it against
something else that fixes the answer.

  - central finite differences of the scalar loss L = sum(dO * O), with O the
    oracle's own forward output, on tiny fp64 inputs (the definition of a
    gradient);
  - torch autograd through the library's scaled_dot_product_attention in
    fp64, dense causal (is_causal) and with explicit masks from a brute-force
    rule set;
  - invariants: each softmax row's score gradients sum to zero, so
    sum_kv dK = 0, and the weights sum to one, so sum_kv dV = sum_q dO;
  - a query with no allowed key contributes nothing and has dQ = 0;
  - the forward half equals the forward oracle.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import Pattern
from test_oracle import rule_sets


def f64(bits):
    return synth.bf16_bits_to_float(bits).astype(np.float64)


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def fd_grads(o, q, k, v, do, p, scale, h=1e-6):
    """Central differences of sum(dO * O) for every element of q, k, v."""
    def loss(q_, k_, v_):
        O = o.attention_bwd(q_, k_, v_, do, p, scale, n_threads=1)[0]
        return float((O * do).sum())

    out = []
    for which in range(3):
        x = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(x[which])
        flat = x[which].reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + h
            lp = loss(*x)
            flat[i] = old - h
            lm = loss(*x)
            flat[i] = old
            g.reshape(-1)[i] = (lp - lm) / (2 * h)
        out.append(g)
    return out


FD_CASES = [
    # (B, Hq, Hkv, N, D, pattern)
    (1, 1, 1, 9, 3, Pattern(window=2, sinks=1)),
    (1, 2, 1, 11, 4, Pattern(window=1, stride=3, n_global=2)),    # GQA: dK, dV sum over the group
    (2, 2, 2, 7, 2, Pattern(window=-1, sinks=2)),                  # sinks only
]


def fd_pin_holds(o, case, tol=1e-7):
    B, Hq, Hkv, N, D, p = case
    q, k, v = rand((B, Hq, N, D), 1), rand((B, Hkv, N, D), 2), rand((B, Hkv, N, D), 3)
    do = rand((B, Hq, N, D), 4)
    scale = 0.7
    _, _, dQ, dK, dV = o.attention_bwd(q, k, v, do, p, scale, n_threads=1)
    gq, gk, gv = fd_grads(o, q, k, v, do, p, scale)
    return all(np.abs(a - b).max() <= tol for a, b in ((dQ, gq), (dK, gk), (dV, gv)))


@pytest.mark.parametrize("case", FD_CASES, ids=lambda c: f"B{c[0]}H{c[1]}/{c[2]}N{c[3]}D{c[4]}")
def test_gradients_match_finite_differences(case):
    assert fd_pin_holds(oracle.default(), case)


def torch_grads(q, k, v, do, scale, mask=None, causal=False):
    """fp64 autograd through the library routine; K, V repeated over the group."""
    group = q.shape[1] // k.shape[1]
    tq, tk, tv = (torch.from_numpy(a).double().requires_grad_(True) for a in (q, k, v))
    O = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(group, 1), tv.repeat_interleave(group, 1),
        attn_mask=None if mask is None else torch.from_numpy(mask), is_causal=causal, scale=scale)
    O.backward(torch.from_numpy(do).double())
    return O.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


def autograd_pin_holds(o, tol=1e-10):
    B, Hq, Hkv, N, D = 1, 4, 2, 48, 16
    q, k, v = (f64(a) for a in synth.qkv(B, Hq, Hkv, N, D, seed=21))
    do = rand((B, Hq, N, D), 5)
    scale = 1 / math.sqrt(D)
    O, _, dQ, dK, dV = o.attention_bwd(q, k, v, do, Pattern(window=N), scale)
    rO, rq, rk, rv = torch_grads(q, k, v, do, scale, causal=True)
    return all(np.abs(a - b).max() <= tol for a, b in ((O, rO), (dQ, rq), (dK, rk), (dV, rv)))


def test_dense_causal_equals_autograd():
    assert autograd_pin_holds(oracle.default())


@pytest.mark.parametrize("p,N", [(Pattern(window=9, sinks=3), 70), (Pattern(window=4, stride=6, n_global=3), 65),
                                 (Pattern(window=0, stride=1), 33)])
def test_masked_equals_autograd_with_explicit_mask(p, N):
    B, Hq, Hkv, D = 2, 2, 1, 8
    q, k, v = (f64(a) for a in synth.qkv(B, Hq, Hkv, N, D, seed=N))
    do = rand((B, Hq, N, D), N)
    mask = np.zeros((N, N), dtype=bool)
    for qi in range(N):
        for kv in rule_sets(N, qi, p):
            mask[qi, kv] = True
    assert mask.any(axis=1).all()  # no empty row: the library routine gives NaN there
    scale = 0.3
    O, _, dQ, dK, dV = oracle.attention_bwd(q, k, v, do, p, scale)
    rO, rq, rk, rv = torch_grads(q, k, v, do, scale, mask=mask)
    for a, b in ((O, rO), (dQ, rq), (dK, rk), (dV, rv)):
        assert np.abs(a - b).max() <= 1e-10


@pytest.mark.parametrize("p", [Pattern(window=20, sinks=4), Pattern(window=5, stride=16, n_global=3)])
def test_gradient_sums(p):
    B, Hq, Hkv, N, D = 2, 4, 2, 150, 8
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=3)
    do = synth.qkv(B, Hq, Hkv, N, D, seed=4)[0]
    _, _, dQ, dK, dV = oracle.attention_bwd(q, k, v, do, p, 0.25)
    assert np.abs(dK.sum(axis=2)).max() <= 1e-10
    dOs = f64(do).reshape(B, Hkv, Hq // Hkv, N, D).sum(axis=(2, 3))
    assert np.abs(dV.sum(axis=2) - dOs).max() <= 1e-10


def test_rows_without_keys_contribute_nothing():
    p = Pattern(window=-1)  # no rule admits any pair: every row is empty
    q, k, v = synth.qkv(1, 2, 1, 40, 8, seed=6)
    do = synth.qkv(1, 2, 1, 40, 8, seed=7)[0]
    O, LSE, dQ, dK, dV = oracle.attention_bwd(q, k, v, do, p, 0.5)
    assert np.all(O == 0) and np.all(np.isneginf(LSE))
    assert np.all(dQ == 0) and np.all(dK == 0) and np.all(dV == 0)


def test_forward_half_equals_forward_oracle():
    for p in (Pattern(window=30, sinks=4), Pattern(window=7, stride=9, n_global=2)):
        q, k, v = synth.qkv(2, 4, 2, 130, 16, seed=8)
        do = synth.qkv(2, 4, 2, 130, 16, seed=9)[0]
        O, LSE, *_ = oracle.attention_bwd(q, k, v, do, p, 0.25)
        O2, LSE2 = oracle.attention(q, k, v, p, 0.25)
        assert np.abs(O - O2).max() <= 1e-12
        assert np.array_equal(np.isneginf(LSE), np.isneginf(LSE2))
        fin = np.isfinite(LSE2)
        assert np.abs(LSE[fin] - LSE2[fin]).max() <= 1e-12
