"""Host check of the exact index steps of tq3_encode_exact (page "tq3_core.py",
_quantize_to_indices: searchsorted(TQ3_BOUNDARIES, xs, right=False), the number of boundaries
strictly below xs). The kernel forms a' = RU(|q| - q 2^-24), counts the positive boundaries b with
b < a' as sat(RN(a' 2^26 - b 2^26)) steps, and takes idx = 4 + c for q > 0, 3 - c otherwise. Each
fp32 operation is evaluated exactly here and rounded once; the index must equal searchsorted for
every boundary's neighbouring fp32 values (both signs), both zeros, powers of two and random
scaled coefficients in [-1, 1].
"""
from fractions import Fraction as Fr

import numpy as np

from fp32emu import fma_f32

B_POS = [float(np.float32(b)) for b in (0.2304, 0.4824, 0.7992)]
BOUNDARIES = sorted([-b for b in B_POS] + [0.0] + B_POS)
M = 2.0 ** 26


def _index(q):
    ap = fma_f32(q, -2.0 ** -24, abs(q), "ru")
    c = 0.0
    for b in B_POS:
        K = float(np.float32(-b * M))
        assert Fr(K) == -Fr(b) * Fr(M)
        c += min(max(fma_f32(ap, M, K, "rn"), 0.0), 1.0)
    assert c in (0.0, 1.0, 2.0, 3.0)
    return int(4 + c) if q > 0.0 else int(3 - c)


def _neighbours(v, k=4):
    out, x = [], np.float32(v)
    for direction in (np.float32(np.inf), np.float32(-np.inf)):
        y = x
        for _ in range(k):
            y = np.nextafter(y, direction, dtype=np.float32)
            out.append(float(y))
    return out + [float(x)]


def test_exact_index_steps_equal_searchsorted():
    qs = {0.0, -0.0, 1.0, -1.0, 1e-45, -1e-45}
    for b in B_POS:
        for v in _neighbours(b):
            qs.update((v, -v))
    for e in range(-10, 1):
        for v in _neighbours(2.0 ** e, 2):
            qs.update((v, -v))
    rng = np.random.default_rng(3)
    qs.update(float(v) for v in rng.uniform(-1, 1, 4000).astype(np.float32))
    for q in qs:
        want = sum(1 for b in BOUNDARIES if b < q)
        assert _index(q) == want, q
