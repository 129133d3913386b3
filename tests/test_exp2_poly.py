"""The FMA-pipe exponential of the forward kernel (exp2_poly_x2), emulated in
float32 on the CPU with the constants read from the kernel source: its
relative error against 2^x stays within the bound the fit reports, it is
exactly 0 below -125 and for -inf, and the constants match a fresh fit."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KERNEL = os.path.join(ROOT, "block_sparse_attention_build_b200", "csrc", "fwd_sm100.cuh")
sys.path.insert(0, os.path.join(ROOT, "block_sparse_attention_build_b200", "csrc"))


def kernel_coefficients():
    src = open(KERNEL).read()
    body = src[src.index("void exp2_poly_x2"):]
    body = body[: body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body)]
    c3, c2, c1, c0 = vals  # Horner order in the source
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def f32(x):
    return np.asarray(x, dtype=np.float32)


def fma32(a, b, c):
    return f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def exp2_poly(x):
    c0, c1, c2, c3 = kernel_coefficients()
    x = f32(x)
    k = np.float32(12582912.0)
    with np.errstate(invalid="ignore", over="ignore"):
        t = f32(x + k)
        j = f32(t - k)
        f = fma32(j, f32(-1.0), x)
        q = fma32(f32(c3), f, f32(c2))
        q = fma32(q, f, f32(c1))
        q = fma32(q, f, f32(c0))
        qi = q.view(np.int32).astype(np.int64)
        ti = t.view(np.int32).astype(np.int64)
        r = ((qi + ((ti << 23) & 0xFFFFFFFF)) & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    return np.where(x < -125.0, np.float32(0.0), r)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-125, 9, 2_000_001), -np.abs(np.random.default_rng(0).normal(0, 20, 100000))])
    x = x[x >= -125]
    got = exp2_poly(x).astype(np.float64)
    ref = np.exp2(f32(x).astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 8e-5


def test_zero_below_range_and_for_neg_inf():
    x = f32([-125.5, -126, -149, -200, -1e30, -np.inf])
    assert np.all(exp2_poly(x) == 0)


def test_constants_match_a_fresh_fit():
    from fit_exp2 import remez
    c, e = remez(3)
    assert e < 8e-5
    assert np.allclose(np.array(kernel_coefficients(), dtype=np.float64), c, rtol=0, atol=1e-6)
