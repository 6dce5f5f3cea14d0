"""Pins of the fixed-order fp32 combine (reading R5): the float32 fused
multiply-add against exact rational arithmetic, and the combine against a
per-element rational evaluation of the same ascending-j recurrence."""
from fractions import Fraction

import numpy as np
import torch

from oracle import moe_oracle as O


def f32_round(v: Fraction) -> Fraction:
    """Nearest float32 of an exact rational (ties to even), normal range."""
    if v == 0:
        return Fraction(0)
    sgn = -1 if v < 0 else 1
    a = abs(v)
    e = 0
    while a >= 2 ** 24:
        a /= 2
        e += 1
    while a < 2 ** 23:
        a *= 2
        e -= 1
    n = a.numerator // a.denominator
    r = a - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sgn * Fraction(n) * Fraction(2) ** e


def test_fma_f32_matches_exact_rounding():
    rng = np.random.default_rng(0)
    n = 4000
    a = rng.standard_normal(n).astype(np.float32)
    b = (rng.standard_normal(n) * np.exp2(rng.integers(-20, 20, n))).astype(np.float32)
    c = (rng.standard_normal(n) * np.exp2(rng.integers(-30, 30, n))).astype(np.float32)
    got = O.fma_f32(a, b, c)
    for i in range(n):
        want = f32_round(Fraction(float(a[i])) * Fraction(float(b[i])) + Fraction(float(c[i])))
        assert Fraction(float(got[i])) == want, i


def test_fma_f32_single_rounding_where_double_rounding_fails():
    # a*b = 2^-24 + 26603*2^-71 exactly (8390653 * 16773127 = 2^47 + 26603), so
    # a*b + 1 lies just above the float32 midpoint 1 + 2^-24. Rounding the sum
    # to float64 first drops the excess and leaves the midpoint itself, which
    # then rounds (to even) down to 1; the one correct rounding goes up to 1 + 2^-23.
    a = np.float32(8390653 * 2.0 ** -23)
    b = np.float32(16773127 * 2.0 ** -48)
    c = np.float32(1.0)
    assert float(a) * 2 ** 23 == 8390653 and float(b) * 2 ** 48 == 16773127
    naive = np.float32(np.float64(a) * np.float64(b) + np.float64(c))
    assert naive == np.float32(1.0)
    got = O.fma_f32(a, b, c)
    assert got == 1 + 2 ** -23
    assert Fraction(float(got)) == f32_round(Fraction(float(a)) * Fraction(float(b)) + 1)


def test_combine_fp32_fma_matches_rational_recurrence():
    rng = np.random.default_rng(1)
    T, k, H = 5, 6, 16
    Y = torch.from_numpy(rng.standard_normal((T, k, H)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    w = rng.random((T, k)).astype(np.float32)
    got = O.combine_fp32_fma(Y, w)
    for t in range(T):
        for h in range(H):
            acc = Fraction(0)
            for j in range(k):
                acc = f32_round(Fraction(float(w[t, j])) * Fraction(float(Y[t, j, h])) + acc)
            want = torch.tensor(float(acc), dtype=torch.float32).to(torch.bfloat16).double().item()
            assert got[t, h] == want, (t, h)
    # within rounding of the float64 combine
    ref = O.combine(Y.astype(np.float64), w)
    assert np.abs(got - ref).max() <= 2 ** -7 * np.abs(ref).max()
