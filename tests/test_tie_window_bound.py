"""The error bound behind the fit kernel's fast code path, checked in exact arithmetic.

The final codes are clamp(rne(fl(X / (rho c)))) (the quotient by the exact
product of the two binary16 scales; hyper.ai summary, Method, symmetric
uniform quantisation to the nearest level).  The kernel first forms the fast
product t = fl(X fl(1/rho)) * r, r a reciprocal of c within 1 ulp of the
correctly rounded one (the exact product t is what its fma rounds), and
takes the IEEE quotient only when t lies within 2^-14 of a rounding tie.
That is exact whenever |t - fl(X / (rho c))| < 2^-14 for |t| <= 127.5 (a
larger |t| is clamped to +-qmax either way); the bound used is
1.5 * 2^-22 |t| (<= 4.6e-5).  This test evaluates both sides with Python
fractions for random binary16 scales (normal and subnormal), every
reciprocal 1 ulp below, at and above the correctly rounded one, and values X
spread over |t| <= 127.5, and checks the bound; and that outside the window
the fast code equals the quotient's.
"""

from fractions import Fraction

import numpy as np

B = Fraction(3, 2) * Fraction(1, 2 ** 22)
WINDOW = Fraction(1, 2 ** 14)


def f32(x) -> Fraction:
    return Fraction(float(np.float32(x)))


def rn32(q: Fraction) -> Fraction:
    """Correct rounding of an exact rational to binary32 (normal range)."""
    if q == 0:
        return Fraction(0)
    s = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp = Fraction(2) ** (e - 23)
    m = a / ulp
    lo = m.numerator // m.denominator
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return s * lo * ulp


def rne(q: Fraction) -> int:
    lo = q.numerator // q.denominator
    rem = q - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 != 0):
        return lo + 1
    return lo


def neighbours(x: Fraction):
    """x and the binary32 values one ulp below and above it (x normal, > 0)."""
    v = np.float32(float(x))
    return [Fraction(float(np.nextafter(v, np.float32(0)))), x,
            Fraction(float(np.nextafter(v, np.float32(np.inf))))]


def test_fast_product_within_bound_of_the_quotient():
    rng = np.random.default_rng(2)
    worst = Fraction(0)
    checked = 0
    for _ in range(300):
        # binary16 scales: a quarter of them subnormal
        rho = Fraction(float(np.float16(np.exp(rng.uniform(-9, 4)))))
        c = Fraction(float(np.float16(np.exp(rng.uniform(-12, 2)) if rng.random() > 0.25
                                      else rng.integers(1, 1024) * 2.0 ** -24)))
        if rho == 0 or c == 0:
            continue
        ir = rn32(1 / rho)
        for r in neighbours(rn32(1 / c)):
            for _ in range(6):
                t_target = Fraction(float(rng.uniform(-127.5, 127.5)))
                X = f32(float(t_target * rho * c))
                if X == 0:
                    continue
                z = rn32(X * ir)
                t = z * r                        # the exact product the fma rounds
                q = rn32(X / (rho * c))          # the quotient the oracle rounds
                if abs(t) > Fraction(255, 2):
                    continue
                err = abs(t - q)
                assert err <= B * abs(t) * (1 + Fraction(1, 2 ** 20)), (rho, c, r, X)
                worst = max(worst, err)
                checked += 1
                # outside the window both sides give the same integer code
                d = t - rne(t)
                if abs(d) <= Fraction(1, 2) - WINDOW:
                    assert rne(t) == rne(q)
    assert checked > 3000
    assert worst < WINDOW
    assert B * Fraction(255, 2) < WINDOW          # 4.6e-5 < 6.1e-5


def test_the_window_catches_constructed_near_ties():
    # X chosen so that the quotient sits exactly on a tie and just beside it:
    # the fast product then lands inside the window, where the kernel takes
    # the IEEE quotient
    rho = Fraction(float(np.float16(0.75)))
    c = Fraction(float(np.float16(0.0312)))
    ir = rn32(1 / rho)
    for k in (0, 3, 30, 126):
        for off in (0, 2 ** -20, -2 ** -20):
            X = f32(float((k + Fraction(1, 2) + Fraction(off)) * rho * c))
            q = rn32(X / (rho * c))
            for r in neighbours(rn32(1 / c)):
                t = rn32(X * ir) * r
                if abs(q - rne(q) - (k + Fraction(1, 2) - rne(q))) < Fraction(1, 2 ** 16):
                    assert abs(t - rne(t)) > Fraction(1, 2) - WINDOW
