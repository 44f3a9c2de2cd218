"""Host check of the exact decision steps the RPBH quantize kernels use for an antisymmetric
codebook (page "orbit_quant.py", _quantize_rows: codes = bucketize(u, edges), right=False, with
edges the fp32 midpoints of the scaled Lloyd-Max codebook).

Instead of comparing u with every edge, the kernels
  * form a' = RU(|u| - u 2^-24): |u| for u > 0 and the next fp32 value above |u| for u < 0, which
    turns the "<=" a negative value needs into a strict compare;
  * count the positive edges below a' with exact 0/1 steps sat(RN(a' M + K)), M = 2^(24 - E)
    (E the edge's binary exponent) and K = -edge M;
  * take the sign of RD(u + (-0)), negative for both zeros;
  * and give the code as the low byte of one rounded sum: 2^23 + mid + 1/2 + sgn (c + 1/2), or, in
    the warp-lane kernel at 3 bits, twice the code as the low byte of the packed
    fma(sgn, c, 2^22 + 3.5).
This test evaluates each of those fp32 operations exactly (rational arithmetic, then the stated
rounding) and checks that the code equals #{k : edge_k < u} for every u tried: every edge, its
neighbouring fp32 values and their negatives, both zeros, subnormals and random directions.
"""
import math
from fractions import Fraction as Fr

import numpy as np
import pytest

from fp32emu import fma_f32, round_f32


def _f32(x):
    return np.float32(x)


_round = round_f32
_fma = fma_f32


def _sat(x):
    return min(max(x, 0.0), 1.0)


def _sign_rd_plus_neg_zero(u):
    """Sign bit of RD(u * 1 + (-0)): an exact zero result takes the sign of round-down, -0."""
    return u < 0 or u == 0.0


def _steps(edges):
    """(M, K) of each positive edge, as the host builds them."""
    out = []
    for e in edges:
        _, ex = math.frexp(e)  # e = f 2^ex, f in [0.5, 1)
        M = math.ldexp(1.0, 25 - ex)
        K = float(_f32(-e * M))
        assert Fr(K) == -Fr(e) * Fr(M)  # exact
        out.append((M, K))
    return out


def _codes(u, pos_edges, steps, bits):
    """The kernel's code of u, both formulations (sym_codes and the warp-lane 3-bit one)."""
    mid = (1 << bits) // 2 - 1
    ap = _fma(u, -2.0 ** -24, abs(u), "ru")
    c = 0.5
    for M, K in steps:
        c += _sat(_fma(ap, M, K, "rn"))  # every partial sum is exact (a half-integer below 8)
    neg = _sign_rd_plus_neg_zero(u)
    sc = -c if neg else c
    v = _round(Fr(_round(Fr(sc) + Fr(0.5), "rn")) + Fr(2 ** 23 + mid), "rn")
    code = int(np.float32(v).view(np.uint32) & 0xFF)
    lanes = None
    if bits == 3:
        w = _fma(-1.0 if neg else 1.0, c, 2.0 ** 22 + 3.5, "rn")
        twice = int(np.float32(w).view(np.uint32) & 0xFF)
        assert twice % 2 == 0
        lanes = twice // 2
    return code, lanes


def _inputs(edges, rng):
    us = {0.0, -0.0, 1e-45, -1e-45, 1e-38, -1e-38, 1.0, -1.0}
    for e in edges:
        x = np.float32(e)
        for k in range(-3, 4):
            y = x
            step = np.float32(np.inf) if k > 0 else np.float32(-np.inf)
            for _ in range(abs(k)):
                y = np.nextafter(y, step, dtype=np.float32)
            us.add(float(y))
            us.add(-float(y))
    scale = max(abs(e) for e in edges) * 1.5
    us.update(float(v) for v in (rng.standard_normal(1500) * scale).astype(np.float32))
    return sorted(us, key=lambda t: (t, math.copysign(1.0, t)))


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [3072, 11008])
def test_exact_steps_equal_bucketize(oracle, bits, d):
    cb = np.asarray(oracle.rpbh_codebook(bits, d), np.float32)
    L = 1 << bits
    edges = [float((cb[k] + cb[k + 1]) / np.float32(2)) for k in range(L - 1)]
    assert all(cb[k] == -cb[L - 1 - k] for k in range(L)) and edges[L // 2 - 1] == 0.0  # antisymmetric
    pos = edges[L // 2:]
    steps = _steps(pos)
    rng = np.random.default_rng(bits * 7 + d)
    for u in _inputs(edges, rng):
        want = sum(1 for e in edges if e < u)  # bucketize(u, edges, right=False)
        code, lanes = _codes(u, pos, steps, bits)
        assert code == want, (bits, d, u)
        if lanes is not None:
            assert lanes == want, (bits, d, u)
