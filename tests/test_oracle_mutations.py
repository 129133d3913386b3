"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that
the pins catch each one: a wrong window bound, sink bound, stride reading, LSE
base, head mapping, missing scale, or tile-fullness test; in the backward, a
dropped softmax row term, a wrong sign, a missing scale, a transposed operand
or a group head left out.  A pin set that let one of these through would not
be pinning the oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import Pattern

from test_oracle import (closed_live_window_sinks, closed_pairs_window_sinks,
                         closed_row_count_strided, rule_sets)
from test_oracle_bwd import FD_CASES, autograd_pin_holds, fd_pin_holds

MUTANTS = {
    "window_exclusive": ("dist <= p->window", "dist < p->window"),
    "sinks_inclusive": ("if (kv < p->sinks)", "if (kv <= p->sinks)"),
    "stride_absolute": ("delta % p->stride == 0", "kv % p->stride == 0"),
    "lse_base2": ("*lse = m + log(l);", "*lse = m + log2(l);"),
    "head_map_modulo": ("int64_t hkv = hq / group;", "int64_t hkv = hq % Hkv;"),
    "scale_dropped": ("bf16_to_double(kp[c]);\n                        s[t] = scale * dot;",
                      "bf16_to_double(kp[c]);\n                        s[t] = dot;"),
    "full_ignores_ragged": ("full[i * T + c] = allowed == (q1 - q0) * (k1 - k0);",
                            "full[i * T + c] = allowed == (int64_t)block * block;"),
    "global_rows_causal_anyway": ("if (p->global_rows_see_all && q < p->n_global)\n        return 1;",
                                  "if (p->global_rows_see_all && q < p->n_global)\n        return delta >= 0;"),
}


def pins_hold(o: oracle.Oracle) -> bool:
    """A compact run of the pins; False as soon as one fails."""
    # printed figure
    counts, _, _ = o.block_mask(Pattern(window=1024, sinks=4), 8192, 128)
    if counts.sum() != 595:
        return False
    # closed forms
    if o.count_pairs(Pattern(window=50, sinks=4), 600) != closed_pairs_window_sinks(600, 50, 4):
        return False
    if o.count_pairs(Pattern(window=10, stride=7, n_global=3), 300) != sum(
            closed_row_count_strided(q, 10, 7, 3) for q in range(300)):
        return False
    counts, _, _ = o.block_mask(Pattern(window=100, sinks=3), 1000, 64)
    if counts.sum() != closed_live_window_sinks(16, 100, 64, 3):
        return False
    # brute force on ragged tiny cases (the second has full ragged tiles)
    for p, N, b in [(Pattern(window=3, sinks=2), 37, 8), (Pattern(window=30, sinks=2), 37, 8)]:
        sets = [rule_sets(N, q, p) for q in range(N)]
        counts, index, full = o.block_mask(p, N, b)
        for i in range(-(-N // b)):
            for c in range(counts[i]):
                j = index[i, c]
                qs = range(i * b, min(N, (i + 1) * b))
                ks = range(j * b, min(N, (j + 1) * b))
                n = sum(1 for q in qs for kv in ks if kv in sets[q])
                if full[i, c] != int(n == len(qs) * len(ks)):
                    return False
    # Q = 0 gives ln |A(q)|
    N, D, w, s = 200, 8, 20, 4
    q = np.zeros((1, 1, N, D), dtype=np.uint16)
    _, k, v = synth.qkv(1, 1, 1, N, D, seed=9)
    _, LSE = o.attention(q, k, v, Pattern(window=w, sinks=s), 0.5)
    cnt = np.array([min(r, w) + 1 + min(s, max(0, r - w)) for r in range(N)])
    if np.abs(LSE[0, 0] - np.log(cnt)).max() > 1e-12:
        return False
    # global rows under the reading that they see every key: closed-form count
    if o.count_pairs(Pattern(window=10, stride=7, n_global=3, global_rows_see_all=1), 300) != 300 * 3 + sum(
            closed_row_count_strided(q, 10, 7, 3) for q in range(3, 300)):
        return False
    # dense causal with GQA equals the library routine
    B, Hq, Hkv, N, D = 1, 4, 2, 64, 16
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=11)
    O, _ = o.attention(q, k, v, Pattern(window=N), 1 / math.sqrt(D))
    f = lambda a: torch.from_numpy(synth.bf16_bits_to_float(a)).double()
    ref = torch.nn.functional.scaled_dot_product_attention(
        f(q), f(k).repeat_interleave(2, 1), f(v).repeat_interleave(2, 1), is_causal=True, scale=1 / math.sqrt(D))
    if np.abs(O - ref.numpy()).max() > 1e-12:
        return False
    return True


def test_unmutated_oracle_passes():
    assert pins_hold(oracle.default())


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = oracle.source()
    assert src.count(old) == 1, f"mutation site for {name} not found"
    path = oracle.compile_source(src.replace(old, new), str(tmp_path / f"lib_{name}.so"))
    assert not pins_hold(oracle.Oracle(path))


NONCAUSAL_MUTANTS = {
    "window_one_sided": ("int64_t dist = delta < 0 ? -delta : delta;", "int64_t dist = delta;"),
    "area_stripe_shifted": ("q / p->area == kv / p->area", "(q + 1) / p->area == kv / p->area"),
    "area_ignored": ("if (p->area > 0 && q / p->area", "if (p->area < 0 && q / p->area"),
    "summary_first_positions": ("kv % p->area >= p->area - p->summary", "kv % p->area < p->summary"),
}


def noncausal_pins_hold(o: oracle.Oracle) -> bool:
    from test_oracle_noncausal import fixed_sets, nc_sets
    N = 37
    for q in range(N):
        for kv in range(N):
            if o.allowed(Pattern(window=-1, causal=1, area=8, summary=2), q, kv) != (kv in fixed_sets(N, q, 8, 2)):
                return False
    if o.count_pairs(Pattern(window=-1, causal=0, area=400), 1600) != 640000:
        return False
    if o.count_pairs(Pattern(window=37, causal=0), 1000) != sum(min(q, 37) + min(999 - q, 37) + 1 for q in range(1000)):
        return False
    if o.count_pairs(Pattern(window=-1, causal=1, area=128, summary=16), 1024) != sum(
            q % 128 + 1 + (q // 128) * 16 for q in range(1024)):
        return False
    for p, N in [(Pattern(window=2, sinks=3, causal=0, area=7), 33), (Pattern(window=-1, causal=1, area=6), 31)]:
        for q in range(N):
            for kv in range(N):
                if o.allowed(p, q, kv) != (kv in nc_sets(N, q, p)):
                    return False
    return True


def test_unmutated_oracle_passes_noncausal_pins():
    assert noncausal_pins_hold(oracle.default())


@pytest.mark.parametrize("name", sorted(NONCAUSAL_MUTANTS))
def test_noncausal_mutant_is_caught(name, tmp_path):
    old, new = NONCAUSAL_MUTANTS[name]
    src = oracle.source()
    assert src.count(old) == 1, f"mutation site for {name} not found"
    path = oracle.compile_source(src.replace(old, new), str(tmp_path / f"lib_{name}.so"))
    assert not noncausal_pins_hold(oracle.Oracle(path))


BWD_MUTANTS = {
    "bwd_dq_delta_dropped": ("double ds = exp(s[t] - lse) * (dp[t] - dl);", "double ds = exp(s[t] - lse) * dp[t];"),
    "bwd_dk_delta_sign": ("double ds = pw * (d - delta[qrow]);", "double ds = pw * (d + delta[qrow]);"),
    "bwd_dk_scale_dropped": ("dk[c] += scale * ds * qv[c];", "dk[c] += ds * qv[c];"),
    "bwd_dv_takes_score_grad": ("dv[c] += pw * dov[c];", "dv[c] += ds * dov[c];"),
    "bwd_dq_uses_values": ("dq[c] += scale * ds * kb[keys[t] * D + c];", "dq[c] += scale * ds * vb[keys[t] * D + c];"),
    "bwd_first_group_head_only": ("for (int64_t hq = hkv * group; hq < (hkv + 1) * group; hq++)",
                                  "for (int64_t hq = hkv * group; hq < hkv * group + 1; hq++)"),
    "bwd_delta_from_values_only": ("dl += pw * d;", "dl += d;"),
}


def bwd_pins_hold(o: oracle.Oracle) -> bool:
    return all(fd_pin_holds(o, c) for c in FD_CASES) and autograd_pin_holds(o)


def test_unmutated_backward_passes():
    assert bwd_pins_hold(oracle.default())


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_backward_mutant_is_caught(name, tmp_path):
    old, new = BWD_MUTANTS[name]
    src = oracle.source()
    assert src.count(old) == 1, f"mutation site for {name} not found"
    path = oracle.compile_source(src.replace(old, new), str(tmp_path / f"lib_{name}.so"))
    assert not bwd_pins_hold(oracle.Oracle(path))
