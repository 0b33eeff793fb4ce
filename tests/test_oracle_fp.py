"""Pins for the oracle's rounding helpers: exact rational round-half-even to fp16."""
from fractions import Fraction

import numpy as np

from oracle.fp import fp16_rne_sat, f32_rne, two_sum_exact


def _exact_fp16(x: float) -> float:
    """Round a double to fp16 with exact rational arithmetic (ties to even), saturating."""
    if x == 0:
        return x
    fx = Fraction(x)
    a = abs(fx)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -14)
    ulp = Fraction(2) ** (e - 10)
    q = a / ulp
    n = q.numerator // q.denominator
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    r = n * ulp
    if r > 65504:
        r = Fraction(65504)
    return float(r) if x > 0 else -float(r)


def test_fp16_rounding_matches_exact_rational():
    rng = np.random.default_rng(1)
    xs = list(rng.standard_normal(3000) * np.exp(rng.uniform(-20, 12, 3000)))
    # halfway points and their neighbours, subnormals, the overflow edge
    for e in (-24, -20, -15, -14, -3, 0, 5, 14):
        for m in (1, 3, 1023, 1025):
            h = float(Fraction(2) ** e * (1 + Fraction(m, 2048)))
            xs += [h, np.nextafter(h, 0), np.nextafter(h, np.inf), -h]
    xs += [65504.0, 65519.99, 65520.0, 1e6, -1e6, 5.9604644775390625e-08, 2.9802322387695312e-08]
    xs = np.array(xs, dtype=np.float64)
    got, bits, over = fp16_rne_sat(xs)
    want = np.array([_exact_fp16(float(x)) for x in xs])
    assert np.array_equal(got, want)
    assert np.array_equal(over, np.abs(xs) >= 65520.0)
    assert np.array_equal(bits.view(np.float16).astype(np.float64), got)


def test_f32_rounding_single_step():
    x = np.array([1 + 2.0 ** -24 + 2.0 ** -50, 1 + 2.0 ** -24, 1 + 3 * 2.0 ** -24])
    # above half -> up; exact half -> even (down); 1.5 ulp -> up to even
    assert np.array_equal(f32_rne(x), np.array([1 + 2.0 ** -23, 1.0, 1 + 2.0 ** -22]))


def test_two_sum_exactness_flag():
    assert two_sum_exact(np.array([1.0]), np.array([2.0 ** -52]))[0]
    assert not two_sum_exact(np.array([1.0]), np.array([2.0 ** -53 * 3]))[0]
