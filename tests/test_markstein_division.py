"""Host check of the division the kernels use where the pages divide (page "tq3_core.py",
tq3_quantize: x / norm and xh / scale in tq3_encode_exact; page "orbit_quant.py", _quantize_rows:
w_rot / (rho + 1e-10)): Markstein's reciprocal and one FMA correction,
    r = RN(1/d),  q0 = RN(x r),  e = RN(x - q0 d)  (one FMA),  q = RN(q0 + e r).
Each step is evaluated exactly and rounded once here. What holds, and what these tests pin:
  * q is the correctly rounded quotient RN(x / d) whenever |x| >= 2^-100 and that quotient is a
    normal fp32 value (the remainder e is then about 2^-24 |x| or more and normal; it is not
    always exact, but the final rounding still is);
  * with smaller numerators or subnormal quotients q can be one unit in the last place of RN(x / d)
    away (a unit never smaller than 2^-149), never of the other sign.
"""
from fractions import Fraction as Fr

import numpy as np

from fp32emu import fma_f32, round_f32

TINY = 2.0 ** -126
SUB_ULP = 2.0 ** -149


def markstein(x, d):
    r = round_f32(Fr(1) / Fr(d), "rn")
    q0 = round_f32(Fr(x) * Fr(r), "rn")
    e = fma_f32(-q0, d, x)
    return fma_f32(e, r, q0)


def _f(v):
    return float(np.float32(v))


def test_correctly_rounded_for_normal_quotients():
    rng = np.random.default_rng(11)
    n = 0
    for _ in range(12000):
        d = _f(np.exp2(rng.uniform(-27, 30)))                          # norms, scales, rho + 1e-10
        x = _f(rng.choice([-1.0, 1.0]) * np.exp2(rng.uniform(-100, 32)))  # elements, rotated values
        want = round_f32(Fr(x) / Fr(d), "rn")
        if abs(want) < TINY:
            continue
        assert markstein(x, d) == want, (x, d)
        n += 1
    for _ in range(3000):  # quotients near 1 (a direction's largest component, x ~ norm)
        d = _f(rng.uniform(0.5, 4.0))
        x = _f(d * rng.uniform(0.999, 1.001))
        assert markstein(x, d) == round_f32(Fr(x) / Fr(d), "rn"), (x, d)
        n += 1
    assert n > 12000
    for d in (1.0, 2.0, 0.5, 1e-8, 3.0, 7.0, 1.0000001):
        for x in (0.0, -0.0, 1.0, -1.0, 3.0, 6.0, -21.0, 1e-30):
            d32, x32 = _f(d), _f(x)
            assert markstein(x32, d32) == round_f32(Fr(x32) / Fr(d32), "rn")


def _ulp(v):
    v = np.float32(abs(v))
    return max(float(np.nextafter(v, np.float32(np.inf), dtype=np.float32) - v), SUB_ULP)


def test_tiny_numerators_at_most_one_unit_off():
    rng = np.random.default_rng(12)
    seen = 0
    for _ in range(6000):
        d = _f(np.exp2(rng.uniform(-27, 30)))
        x = _f(rng.choice([-1.0, 1.0]) * np.exp2(rng.uniform(-150, -90)))
        got, want = markstein(x, d), round_f32(Fr(x) / Fr(d), "rn")
        if got != want:
            seen += 1
            assert abs(got - want) <= _ulp(want) and got * want >= 0, (x, d, got, want)
    assert seen > 0  # the deviation is real, so the reading must stay documented
