"""Pins of the oracle's attention with bf16-rounded softmax weights (round_p).

The rounding point of P is a reading, not something the pages fix (DFlash-ja
section 2.2, parallel block diffusion bullet, says only that one pass attends
over the injected context and the block).  The reading: t_i = q.k_i log2(e) /
sqrt(d), B = floor(max t), P_i = R(2^(t_i - B)), o = sum P_i v_i / sum 2^(t_i - B).

Pinned here, independently of the oracle's own code:
  * hand-worked cases (tests/golden/attention_bf16p.txt) whose weights sit on
    both sides of bf16 rounding ties, with the expected P, Z and o as exact
    rationals; the hand-rounded values are themselves checked by brute force;
  * plausible mistakes (rounding P/Z instead of P, the exact maximum instead of
    its floor, a rounded denominator, no rounding) all miss the golden values;
  * split invariance: keys cut into blocks, each with its own integer base,
    merged by exact powers of two, give bit-identical rounded numerators and
    the same denominator as one pass over all keys.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "attention_bf16p.txt")
D = 16   # head_dim of the golden cases: sqrt(d) = 4 exactly


def _frac(expr: str) -> Fraction:
    """'a/b+c/d-e/f*g/h' with +, -, * over integers and fractions (left to right for * within a term)."""
    total = Fraction(0)
    term, sign, i = "", 1, 0
    parts = []
    for ch in expr:
        if ch in "+-" and term:
            parts.append((sign, term))
            term, sign = "", (1 if ch == "+" else -1)
        elif ch in "+-":
            sign = 1 if ch == "+" else -1
        else:
            term += ch
    parts.append((sign, term))
    for sign, t in parts:
        v = Fraction(1)
        for f in t.split("*"):
            v *= Fraction(f)
        total += sign * v
    return total


def _cases():
    out = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, b, ms, rs = [x.strip() for x in line.split("|")]
            m = [_frac(x) for x in ms.split()]
            r = [_frac(x) for x in rs.split()]
            assert len(m) == len(r)
            out.append((name, int(b), m, r))
    return out


CASES = _cases()


def _bf16_neighbours(x: Fraction):
    """The bf16 values just below and just above x > 0 (8 significant bits)."""
    e = math.floor(math.log2(x))
    while Fraction(2) ** e > x:
        e -= 1
    while Fraction(2) ** (e + 1) <= x:
        e += 1
    step = Fraction(2) ** (e - 7)
    lo = (x // step) * step
    return lo, lo + step


def test_golden_file_rounding_is_nearest_even_by_brute_force():
    assert len(CASES) == 4
    for name, _, m, r in CASES:
        for mi, ri in zip(m, r):
            lo, hi = _bf16_neighbours(mi)
            if mi == lo:
                assert ri == mi, name
                continue
            dlo, dhi = mi - lo, hi - mi
            assert dlo != dhi, (name, "exact tie in a golden case")
            assert ri == (lo if dlo < dhi else hi), (name, mi, ri)
            # every weight is well away from a tie (relative 2^-14)
            tie = (lo + hi) / 2
            assert abs(mi - tie) / mi >= Fraction(1, 2 ** 14), (name, mi)


def _inputs(B: int, m):
    """One query row, one head, head_dim 16: keys with t_i = B + log2(m_i), one-hot values."""
    n = len(m)
    q = np.zeros((1, 1, D))
    q[0, 0, 0] = 1.0
    k = np.zeros((1, n, D))
    v = np.zeros((1, n, D))
    for i, mi in enumerate(m):
        t = B + math.log2(float(mi))
        k[0, i, 0] = t * math.sqrt(D) * math.log(2.0)     # t = k . q * log2(e) / sqrt(d)
        v[0, i, i] = 1.0
    return q, k, v


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_attention_round_p_matches_hand_worked_case(case):
    name, B, m, r = case
    q, k, v = _inputs(B, m)
    n = len(m)
    Z = sum(m)
    num, z, base = O.attention_block(q, k, v, round_p=True)
    assert base[0, 0] == B
    # P_i lands exactly on the hand-rounded value
    assert [Fraction(x) for x in num[0, 0, :n]] == r, (name, num[0, 0, :n])
    assert z[0, 0] == pytest.approx(float(Z), rel=1e-14)
    o = O.attention(q, k, v, round_p=True)
    want = np.array([float(ri / Z) for ri in r])
    assert np.allclose(o[0, 0, :n], want, rtol=1e-13, atol=0)
    assert np.all(o[0, 0, n:] == 0)


# --- plausible mistakes, planted in a plain numpy restatement of the weights -------
def _r_bf16(x):
    return torch.tensor(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


def _mutant(t, kind):
    mx = t.max()
    if kind == "exact_max":
        e = np.exp2(t - mx)
        return _r_bf16(e) / e.sum()
    e = np.exp2(t - math.floor(mx))
    if kind == "round_after_normalising":
        return _r_bf16(e / e.sum())
    if kind == "rounded_denominator":
        return _r_bf16(e) / _r_bf16(e).sum()
    if kind == "no_rounding":
        return e / e.sum()
    raise KeyError(kind)


@pytest.mark.parametrize("kind", ["exact_max", "round_after_normalising", "rounded_denominator", "no_rounding"])
def test_plausible_mistakes_miss_the_golden_values(kind):
    missed = 0
    for name, B, m, r in CASES:
        t = np.array([B + math.log2(float(mi)) for mi in m])
        want = np.array([float(ri / sum(m)) for ri in r])
        got = _mutant(t, kind)
        if not np.allclose(got, want, rtol=1e-9, atol=0):
            missed += 1
    # each mistake is caught by at least one hand-worked case
    assert missed >= 1, kind


def test_round_p_split_invariance_bit_exact():
    """Blocks of keys with their own integer bases, merged by exact powers of two,
    reproduce the one-pass rounded numerators bit for bit (values are small
    integers and weights stay above 2^-20, so every fp64 sum is exact) and the
    one-pass denominator to rounding."""
    rng = np.random.default_rng(12345)
    nrow, nq, nkv, d, n = 4, 4, 2, 64, 300
    q = rng.standard_normal((nrow, nq, d)) * 0.5
    k = rng.standard_normal((nkv, n, d)) * 0.5
    v = rng.integers(-100, 101, size=(nkv, n, d)).astype(np.float64)
    scale = math.log2(math.e) / math.sqrt(d)
    # scores spread below 20 powers of two: |q.k| scale stays well inside that
    t = np.einsum("rhd,gnd->rhgn", q, k) * scale
    assert t.max() - t.min() < 20
    num1, z1, b1 = O.attention_block(q, k, v, round_p=True)
    for cuts in ([0, 64, 128, 300], [0, 7, 150, 151, 299, 300], [0, 1, 300]):
        parts = [O.attention_block(q, k[:, a:b], v[:, a:b], round_p=True) for a, b in zip(cuts[:-1], cuts[1:])]
        bases = np.stack([p[2] for p in parts])            # [blocks, nrow, nq]
        ball = bases.max(axis=0)
        assert np.array_equal(ball, b1)
        num = np.zeros_like(num1)
        z = np.zeros_like(z1)
        for (nb, zb, bb) in parts:
            s = np.ldexp(1.0, (bb - ball).astype(np.int64))
            num += nb * s[..., None]
            z += zb * s
        assert np.array_equal(num, num1), np.max(np.abs(num - num1))
        assert np.allclose(z, z1, rtol=n * 2.0 ** -52, atol=0)   # the same 300 terms, regrouped
        o_split = num / z[..., None]
        o_one = O.attention(q, k, v, round_p=True)
        assert np.allclose(o_split, o_one, rtol=1e-14, atol=1e-14)
