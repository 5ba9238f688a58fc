"""The quotient method of the quantization kernels, checked on the host in exact
arithmetic: with r = RN(1/m), q = RN(w r), e = RN(w - q m) and x = RN(q + e r) (the last
two as fused multiply-adds: one rounding each), x is the correctly rounded fp32 quotient
w / m (P. Markstein, IBM J. Res. Dev. 34, 1990). Level 1 takes x = fl32(w / absmax) this
way and the double quantization y = fl32(cc / c1); both keep plain IEEE division for a
divisor below 2^-64. The check covers |w| <= m (the only quotients either kernel forms)
with m >= 2^-64, and requires the exact quotient wherever |w / m| > 2^-36 (below that,
both kernels' code searches land on the entry of zero whatever the last bit)."""
from fractions import Fraction

import numpy as np

from oracle import nf4_oracle as O


def _rn(x: Fraction) -> np.float32:
    """RN to fp32 of any rational (sign handled around the oracle's rounding)."""
    if x < 0:
        return np.float32(-O.f32_round(-x))
    return O.f32_round(x)


def _fma(a, b, c) -> np.float32:
    return _rn(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def _quot(w, m) -> np.float32:
    r = _rn(Fraction(1) / Fraction(float(m)))
    q = _rn(Fraction(float(w)) * Fraction(float(r)))
    e = _fma(-q, m, w)
    return _fma(e, r, q)


def _cases(rng, n):
    out = []
    for _ in range(n):
        m = np.float32(np.ldexp(1.0 + rng.random(), int(rng.integers(-64, 40))))
        kind = rng.integers(0, 6)
        if kind == 0:
            w = m                                    # x = 1
        elif kind == 1:
            w = np.float32(-m)
        elif kind == 2:                              # the neighbours of m
            w = np.nextafter(m, np.float32(0), dtype=np.float32)
        elif kind == 3:                              # small quotients
            w = np.float32(m * np.float32(np.ldexp(rng.random(), -int(rng.integers(0, 36)))))
        else:
            w = np.float32(m * np.float32(rng.uniform(-1.0, 1.0)))
        if abs(float(w)) <= float(m):
            out.append((w, m))
    # divisors whose significand is all ones or a power of two, and the smallest allowed
    for m in (np.float32(np.ldexp(2.0 - 2.0 ** -23, -3)), np.float32(0.5),
              np.float32(2.0 ** -64), np.float32(np.ldexp(2.0 - 2.0 ** -23, -64))):
        for f in (1.0, -1.0, 0.999999, 0.5000001, 1.0 / 3.0, -0.7071068, 2.0 ** -30):
            out.append((np.float32(m * np.float32(f)), m))
    return out


def test_markstein_quotient_is_correctly_rounded():
    rng = np.random.default_rng(2024)
    bad = []
    for w, m in _cases(rng, 3000):
        exact = _rn(Fraction(float(w)) / Fraction(float(m)))
        got = _quot(w, m)
        if abs(float(w)) > float(m) * 2.0 ** -36 and got != exact:
            bad.append((float(w), float(m), float(got), float(exact)))
    assert not bad, bad[:5]


def test_plain_division_pin():
    """The exact-rational helper itself against IEEE fp32 division by numpy."""
    rng = np.random.default_rng(7)
    for _ in range(500):
        w = np.float32(rng.uniform(-1, 1))
        m = np.float32(rng.uniform(0.01, 3))
        assert _rn(Fraction(float(w)) / Fraction(float(m))) == np.float32(w / m)
