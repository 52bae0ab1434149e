"""Arithmetic identities the quantize kernel relies on, checked on the host.

The kernel's hot path computes rint(fl(v / scale)) for bf16 v and fp16 scale
without a division: q0 = fl(v * rcp), r = v - q0 * scale (one fma, exact),
q1 = fl(q0 + r * rcp) (one fma) with rcp = fl(1 / scale).  That q1 is the
correctly rounded binary32 quotient (P. Markstein's correction step, 1990)
is checked here exhaustively over every pair of significands; the result is
invariant under power-of-two scaling of either operand, so this covers all
normal-range inputs.  The AWQ-scaled path instead brackets the quotient
between v*rcp*(1 - 2^-18) and v*rcp*(1 + 2^-18) and repairs exact ties with
a zero-residual test; both facts are checked on sampled and constructed
inputs with exact rational arithmetic.
"""
from fractions import Fraction

import numpy as np


def _rn32(x64):
    """float64 -> binary32, round to nearest even (numpy's conversion)."""
    return np.asarray(x64, dtype=np.float64).astype(np.float32)


def _rn32_of_sum(a, b):
    """Correctly rounded binary32 value of a + b for float64 arrays a, b with
    |a| >= |b| (the float64 sum may round; its error is recovered exactly with
    Fast2Sum and decides the cases that fall on a binary32 midpoint)."""
    s = a + b
    err = (a - s) + b
    f = _rn32(s).astype(np.float64)
    # spacing of binary32 at |s| (s in the normal range here)
    e = np.floor(np.log2(np.abs(s)))
    ulp = np.exp2(e - 23)
    mid = np.abs(s - f) == ulp / 2
    up = mid & (err != 0) & (np.sign(err) == np.sign(s - f))
    down = mid & (err != 0) & (np.sign(err) != np.sign(s - f))
    # at a midpoint with a nonzero error the true value is on err's side
    g = np.where(up, s + np.sign(s - f) * ulp / 2, f)
    g = np.where(down, s - np.sign(s - f) * ulp / 2, g)
    return g


def _rn32_ratio(num, den):
    """Correctly rounded binary32 of positive integer ratios num/den (int64
    arrays, ratio in [0.5, 2)), as float64."""
    e = np.where(num >= den, 0, -1)
    scaled = num << (23 - e)          # num * 2^(23 - e)
    m = scaled // den
    rem = scaled - m * den
    up = (2 * rem > den) | ((2 * rem == den) & (m % 2 == 1))
    m = m + up
    return m.astype(np.float64) * np.exp2(e - 23.0)


def test_correction_step_is_correctly_rounded_for_bf16_over_fp16():
    mx = np.arange(128, 256, dtype=np.int64)            # bf16 significands
    ms = np.arange(1024, 2048, dtype=np.int64)          # fp16 significands
    MX, MS = np.meshgrid(mx, ms, indexing="ij")
    x = MX.astype(np.float64) / 128.0
    s = MS.astype(np.float64) / 1024.0
    rcp = _rn32(1.0 / s).astype(np.float64)
    # 1/s rounded once: check against exact integer rounding of 1024/ms
    assert np.array_equal(rcp, _rn32_ratio(np.full_like(MS, 1024), MS))
    q0 = _rn32(x * rcp).astype(np.float64)                # product exact in f64
    r = _rn32(x - q0 * s).astype(np.float64)              # residual exact in f64
    q1 = _rn32_of_sum(q0, r * rcp)                        # r*rcp exact in f64
    exact = _rn32_ratio(8 * MX, MS)                       # x/s = 8 mx / ms
    bad = np.flatnonzero(q1 != exact)
    assert bad.size == 0, f"{bad.size} significand pairs differ"


def _f32(v):
    return Fraction(float(np.float32(v)))


def _rn32_frac(v):
    return Fraction(float(np.float32(float(v)))) if abs(v) > Fraction(1, 1 << 100) else Fraction(0)


def test_bracket_contains_quotient_and_tie_test():
    """For binary32 v (as AWQ-scaled values are) and fp16 scales: v*rcp_lo and
    v*rcp_hi strictly bracket both v/scale and fl(v/scale); where the bracket
    holds a half-integer T, v == T*scale exactly iff v - T*scale is zero."""
    rng = np.random.default_rng(7)
    scales = rng.uniform(1e-4, 2e-2, 400).astype(np.float16).astype(np.float32)
    cases = 0
    for sc in scales:
        rcp = np.float32(1.0) / sc
        rh = np.float32(rcp * np.float32(1.0 + 2.0 ** -18))
        rl = np.float32(rcp * np.float32(1.0 - 2.0 ** -18))
        ks = rng.integers(-9, 9, 6)
        # values on exact ties, next to them, and random
        vals = [np.float32((k + 0.5) * float(sc)) for k in ks]
        vals += [np.nextafter(v, np.float32(np.inf)) for v in vals]
        vals += list(rng.normal(0, 8 * float(sc), 6).astype(np.float32))
        S = _f32(sc)
        for v in vals:
            V = _f32(v)
            if V == 0:
                continue
            q = V / S
            fq = Fraction(float(np.float32(v) / sc))   # binary32 division, correctly rounded
            lo, hi = sorted((V * _f32(rl), V * _f32(rh)))
            assert lo < min(q, fq) and max(q, fq) < hi
            a = np.float32(float(V * _f32(rh) + 12582912))  # one rounding of the exact sum
            z = np.float32(float(V * _f32(rl) + 12582912))
            if a != z:
                cases += 1
                assert abs(float(a) - float(z)) == 1.0
                t = Fraction(float(min(a, z))) - 12582912 + Fraction(1, 2)
                assert (V - t * S == 0) == (q == t)
    assert cases > 0
