"""The NVFP4 kernel decides E2M1 codes from two bracketing products and, when
the bracket contains a midpoint M, from the residual |x| - eff * M computed by
one fused multiply-add. This checks that rule on the CPU, in exact rational
arithmetic, against the oracle's E2M1(fl32(x / eff)):

* the residual is exactly representable in fp32 whenever the bracket
  straddles a midpoint (so the hardware FMA returns it exactly), and
* comparing it with eff times half an ulp of M gives the oracle's code,
  including exact ties (x / eff == M), for bf16- and fp32-like numerators.
"""
from fractions import Fraction

import numpy as np

MID = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
EXP = [-2, -1, 0, 0, 1, 1, 2]


def f32(v):
    return float(np.float32(v))


def resolve(x, eff, c):
    """The kernel's rule (e2m1_resolve), with the residual taken exactly."""
    M, eM = MID[c], EXP[c]
    h_above = f32(eff * 2.0 ** (eM - 24))
    h_below = f32(h_above * 0.5) if c == 0 else h_above
    exact = Fraction(abs(x)) - Fraction(eff) * Fraction(M)
    D = f32(float(exact))
    assert Fraction(D) == exact, ("residual not representable", x, eff, c)
    mag = c + 1 if D > h_above else (c if D < -h_below else (c + 1 if c & 1 else c))
    return mag | (8 if np.signbit(x) else 0)


def test_bracket_and_tie_rule_match_oracle(orc):
    rng = np.random.default_rng(0)
    straddled = 0
    for _ in range(30000):
        c = int(rng.integers(0, 7))
        eff = f32(np.exp2(rng.uniform(-90, 90)) * rng.uniform(1, 2))
        base = np.array([np.float32(eff * MID[c])], np.float32).view(np.uint32)[0]
        if rng.random() < 0.5:      # fp32-like numerator within a few ulps
            xb = np.uint32(int(base) + int(rng.integers(-3, 4)))
        else:                       # bf16-like numerator (8 significant bits)
            xb = np.uint32((int(base) & 0xFFFF0000) + (int(rng.integers(0, 3)) << 16))
        x = float(np.array([xb], np.uint32).view(np.float32)[0]) * (1 if rng.random() < 0.5 else -1)
        want = orc.e2m1_encode(float(np.float32(np.float32(x) / np.float32(eff))))
        r = 1.0 / eff
        lo = f32(x * f32(r * 0.99999904632568359375))
        hi = f32(x * f32(r * 1.00000095367431640625))
        cl, ch = orc.e2m1_encode(lo), orc.e2m1_encode(hi)
        if cl == ch:
            assert cl == want
            continue
        straddled += 1
        assert resolve(x, eff, min(cl & 7, ch & 7)) == want, (x, eff, c)
    assert straddled > 10000
