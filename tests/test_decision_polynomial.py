"""Host checks of the constants the fast TQ3 encoders decide with (page "tq3_core.py",
_quantize_to_indices: searchsorted against TQ3_BOUNDARIES, right=False).

Both fast encoders (the tensor-core one for bf16 input, the one-thread-per-vector one for fp32)
compute the index of a scaled coefficient x in [-1, 1] as 3 + ceil(Q(x)),
Q(x) = q1 x + q3 x^3 + q5 x^5, with the three fp32 coefficients written in the shared TQ3 header. These tests
read the coefficients from the source and check, in fp32 arithmetic emulated with numpy, what that
rule relies on: Q passes through 1, 2, 3 at the positive boundaries, is odd and increasing, stays
below 4 at x = 1, and its evaluation (Horner in x^2, the last step an exact product followed by
ceil) reproduces #{j : B_j < x} everywhere except within 2e-7 of a boundary.
"""
import os
import re

import numpy as np

from conftest import ROOT

SRC = os.path.join(ROOT, "weight_quantization_b200", "csrc", "tq3_common.cuh")
B = np.array([-0.7992, -0.4824, -0.2304, 0.0, 0.2304, 0.4824, 0.7992], dtype=np.float32).astype(np.float64)


def _coefs():
    text = open(SRC).read()
    m = re.search(r"k == 1 \? (0x[0-9a-f]+)u : k == 3 \? (0x[0-9a-f]+)u : (0x[0-9a-f]+)u", text)
    assert m, "decision coefficients not found in the encoder source"
    return [np.array([int(h, 16)], np.uint32).view(np.float32)[0] for h in m.groups()]


def _index(x32, q1, q3, q5):
    """3 + ceil(h x) with h = (q5 x^2 + q3) x^2 + q1 in fp32 (each fma rounded once), as the kernel."""
    def fma(a, b, c):
        return (np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64)).astype(np.float32)
    x2 = (x32 * x32).astype(np.float32)
    h = fma(fma(q5, x2, q3), x2, q1)
    return 3 + np.ceil(h.astype(np.float64) * x32.astype(np.float64))


def test_polynomial_interpolates_the_boundaries_and_is_increasing():
    q1, q3, q5 = (np.float64(c) for c in _coefs())
    Q = lambda x: q1 * x + q3 * x ** 3 + q5 * x ** 5
    for k, b in enumerate(B[4:]):
        assert abs(Q(b) - (k + 1)) < 2e-6
    x = np.linspace(-1, 1, 200001)
    assert (q1 + 3 * q3 * x ** 2 + 5 * q5 * x ** 4).min() > 1.9
    assert 3.4 < Q(1.0) < 3.5 and Q(-1.0) == -Q(1.0)


def test_index_rule_matches_searchsorted_outside_a_narrow_band():
    q1, q3, q5 = _coefs()
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-1, 1, 400000), np.repeat(B, 40000) + rng.uniform(-2e-6, 2e-6, 280000),
                        [-1.0, 1.0, 0.0, -0.0, 1e-30, -1e-30, 1e-45, -1e-45]]).astype(np.float32)
    got = _index(x, q1, q3, q5)
    want = np.searchsorted(B, x.astype(np.float64), side="left")
    assert got.min() >= 0 and got.max() <= 7
    bad = got != want
    dist = np.min(np.abs(x[bad].astype(np.float64)[:, None] - B[None, :]), axis=1) if bad.any() else np.zeros(1)
    assert dist.max() < 2e-7, dist.max()
    # exact zeros take the lower bucket, as searchsorted(right=False) gives for 0.0
    assert np.all(got[x == 0] == 3)
    # at a boundary value itself either neighbouring bucket is inside the tie window
    Bf = B.astype(np.float32)
    d = _index(Bf, q1, q3, q5) - np.arange(7)
    assert np.all((d == 0) | (d == 1))
