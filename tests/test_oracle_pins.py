"""Pins for the oracle: each check ties it to something other than itself -- values the pages
print, closed forms, textbook tables, library routines and brute force -- so that a dropped term,
a wrong sign or index, or a transposed operand anywhere in it fails at least one test.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from weight_quantization_b200 import inputs


def golden_dict(name):
    out = {}
    for parts in read_golden(name):
        out[parts[0]] = parts[1:]
    return out


# ------------------------------------------------------------------------------------------
# TQ3 tables ("tq3_core.py": TQ3_CENTROIDS, TQ3_BOUNDARIES)
# ------------------------------------------------------------------------------------------
def test_tq3_tables_match_printed_values(oracle):
    g = golden_dict("tq3_codebook.txt")
    c, b = oracle.tq3_tables()
    assert np.array_equal(c, np.array([float(v) for v in g["centroids"]], np.float32))
    assert np.array_equal(b, np.array([float(v) for v in g["boundaries"]], np.float32))


def test_tq3_boundaries_are_centroid_midpoints(oracle):
    c, b = oracle.tq3_tables()
    mid = (c[:-1].astype(np.float64) + c[1:].astype(np.float64)) / 2
    err = np.abs(mid - b)
    # five boundaries are the midpoints to fp32 rounding; the printed +-0.4824 sit 5e-5 from the
    # midpoint +-0.48235 (the page prints 4 decimals)
    assert np.sum(err < 1e-7) == 5
    assert err.max() <= 5.01e-5
    assert np.all(np.diff(b) > 0) and np.all(np.diff(c) > 0)
    assert np.array_equal(c, -c[::-1]) and np.array_equal(b, -b[::-1])


def test_tq3_bucketize_tie_rule(oracle):
    """searchsorted(right=False): a value equal to a boundary takes the lower index."""
    _, b = oracle.tq3_tables()
    for j, bj in enumerate(b):
        assert oracle.tq3_bucketize(bj) == j
        assert oracle.tq3_bucketize(np.nextafter(bj, np.float32(2))) == j + 1
        assert oracle.tq3_bucketize(np.nextafter(bj, np.float32(-2))) == j
    assert oracle.tq3_bucketize(0.0) == 3 and oracle.tq3_bucketize(-0.0) == 3
    assert oracle.tq3_bucketize(-1.0) == 0 and oracle.tq3_bucketize(1.0) == 7


def test_tq3_bucketize_matches_library_searchsorted(oracle):
    _, b = oracle.tq3_tables()
    v = np.concatenate([inputs.gaussian((4000,), seed=11) * 0.5, b, -b, [0.0, 1.0, -1.0]]).astype(np.float32)
    ref = np.searchsorted(b, v, side="left")
    got = np.array([oracle.tq3_bucketize(x) for x in v])
    assert np.array_equal(ref, got)


def test_tq3_bucketize_vs_nearest_centroid(oracle):
    """Brute-force nearest centroid agrees with the boundary bucketize except on the midpoints
    themselves (equidistant up to fp32 rounding of the centroids) and in the 5e-5 band where the
    printed +-0.4824 differ from the true midpoints."""
    c, b = oracle.tq3_tables()
    v = np.linspace(-1, 1, 20001).astype(np.float32)
    mismatches = 0
    for x in v:
        i = oracle.tq3_bucketize(x)
        k = oracle.nearest_centroid(x, c)
        if i != k:
            mismatches += 1
            assert abs(i - k) == 1
            assert np.min(np.abs(b - x)) < 1e-6 or abs(abs(float(x)) - 0.48235) <= 6e-5
    assert mismatches < 20


# ------------------------------------------------------------------------------------------
# Hadamard ("tq3_core.py" _fwht_inplace, "orbit_quant.py" _fwht)
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64, 128, 1024])
def test_sylvester_hadamard_is_orthogonal(oracle, n):
    H = oracle.hadamard_dense(n).astype(np.int64)
    assert np.array_equal(H @ H, n * np.eye(n, dtype=np.int64))


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 128])
def test_fwht_butterfly_equals_dense_product(oracle, n):
    """With post = 1 and small integers every fp32 sum is exact: the butterfly must equal H @ x."""
    H = oracle.hadamard_dense(n).astype(np.int64)
    x = (inputs.uniform_int((n,), 200, seed=n).astype(np.int64) - 100)
    got = oracle.fwht(x.astype(np.float32), post=1.0)
    assert np.array_equal(got.astype(np.int64), H @ x)


def test_fwht_post_constants(oracle):
    # 1/sqrt(128) rounded to fp32, and h ** -0.5 (exact powers of two for h = 256, 1024)
    assert np.float32(oracle.lib().or_tq3_fwht_post(128)).view(np.uint32) == 0x3DB504F3
    assert oracle.lib().or_rpbh_fwht_post(256) == 0.0625
    assert oracle.lib().or_rpbh_fwht_post(1024) == 2.0 ** -5


def test_fwht_preserves_norm_and_is_self_inverse(oracle):
    g = golden_dict("page_numbers.txt")
    x = inputs.gaussian((8, 128), seed=123)
    errs = []
    for row in x:
        y = oracle.fwht(row)
        assert abs(np.linalg.norm(y.astype(np.float64)) / np.linalg.norm(row.astype(np.float64)) - 1) < 1e-6
        errs.append(np.abs(oracle.fwht(y) - row).max())
    assert max(errs) < float(g["fwht_self_inverse_max_err"][0])


# ------------------------------------------------------------------------------------------
# packing ("tq3_core.py" _pack_3bit/_unpack_3bit, "orbit_quant.py" pack_codes/unpack_codes)
# ------------------------------------------------------------------------------------------
def test_pack_worked_examples(oracle):
    for parts in read_golden("pack_examples.txt"):
        if parts[0] == "tq3":
            name, hexgroup = parts[1], parts[2]
            if name == "ramp0to7":
                idx = np.tile(np.arange(8, dtype=np.uint8), 16)
            elif name == "all3":
                idx = np.full(128, 3, np.uint8)
            else:
                idx = np.full(128, 7, np.uint8)
            packed = oracle.tq3_pack(idx)[0]
            assert packed.size == 48
            assert packed.tobytes() == bytes.fromhex(hexgroup) * 16
            assert np.array_equal(oracle.tq3_unpack(packed)[0], idx)
        else:
            bits = int(parts[1])
            codes = np.array([int(v) for v in parts[2].split(",")], np.uint8)
            packed = oracle.pack_codes(codes, bits)
            assert packed.tobytes() == bytes.fromhex(parts[3])
            assert np.array_equal(oracle.unpack_codes(packed, bits, codes.size), codes)


def test_tq3_pack_roundtrip_random(oracle):
    idx = inputs.uniform_int((16, 128), 8, seed=5)
    assert np.array_equal(oracle.tq3_unpack(oracle.tq3_pack(idx)), idx)


def test_tq3_pack_is_lsb_first_stream(oracle):
    """_pack_3bit equals an LSB-first bitstream with index k at stream bits 3k..3k+2 (numpy)."""
    idx = inputs.uniform_int((3, 128), 8, seed=6)
    bitmat = ((idx[..., None] >> np.arange(3)) & 1).astype(np.uint8).reshape(3, 384)
    ref = np.packbits(bitmat, axis=1, bitorder="little")
    assert np.array_equal(oracle.tq3_pack(idx), ref)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("numel", [1, 7, 8, 13, 1000])
def test_rpbh_pack_matches_numpy_packbits(oracle, bits, numel):
    codes = inputs.uniform_int((numel,), 1 << bits, seed=numel * 10 + bits)
    bitmat = ((codes[:, None] >> np.arange(bits - 1, -1, -1)) & 1).astype(np.uint8).reshape(-1)
    pad = (-numel) % 8 * bits
    ref = np.packbits(np.concatenate([bitmat, np.zeros(pad, np.uint8)]))
    got = oracle.pack_codes(codes, bits)
    assert got.size == (numel + 7) // 8 * bits
    assert np.array_equal(got, ref)
    assert np.array_equal(oracle.unpack_codes(got, bits, numel), codes)


def test_tq3_memory_bytes(oracle):
    g = golden_dict("page_numbers.txt")
    shape = [int(v) for v in g["ltx_shape"]]
    comp, orig, ratio = oracle.tq3_memory_bytes(shape)
    assert comp == int(g["ltx_tq3_bytes"][0]) and orig == int(g["ltx_fp16_bytes"][0])
    comp, orig, ratio = oracle.tq3_memory_bytes([4, 32, 512])
    assert comp == 4 * 32 * 4 * 56 and ratio > float(g["min_compression_ratio"][0])
    assert abs(ratio - 256 / 56) < 1e-12
    with pytest.raises(ValueError):
        oracle.tq3_memory_bytes([4, 100])


# ------------------------------------------------------------------------------------------
# TQ3 encode/decode ("tq3_core.py" tq3_quantize / tq3_dequantize)
# ------------------------------------------------------------------------------------------
def _dense_encode_f64(x, signs):
    """float64 dense restatement (no butterflies) of the encoder's real-valued pipeline."""
    H = np.array([[(-1) ** bin(i & j).count("1") for j in range(128)] for i in range(128)], np.float64)
    x = x.astype(np.float64)
    n = np.maximum(np.linalg.norm(x, axis=1, keepdims=True), 1e-8)
    xh = (x / n * signs) @ H.T / math.sqrt(128)
    s = np.maximum(np.abs(xh).max(axis=1, keepdims=True), 1e-8)
    return xh / s, n[:, 0], s[:, 0], H


def test_tq3_encode_matches_dense_float64(oracle):
    bits = inputs.tq3_sign_bits()
    signs = oracle.tq3_signs(bits).astype(np.float64)
    x = inputs.gaussian((64, 128), seed=21) * 3.0
    xs, idx, norms, scales = oracle.tq3_encode_debug(x, bits)
    xs_ref, n_ref, s_ref, _ = _dense_encode_f64(x, signs)
    assert np.allclose(norms, n_ref, rtol=1e-7, atol=0)
    assert np.allclose(scales, s_ref, rtol=2e-6, atol=0)
    assert np.abs(xs - xs_ref).max() < 2e-6
    # indices: bucketize of the float64 values, except within 2e-6 of a boundary
    _, b = oracle.tq3_tables()
    ref_idx = np.searchsorted(b.astype(np.float64), xs_ref, side="left")
    near = np.min(np.abs(xs_ref[..., None] - b.astype(np.float64)), axis=-1) < 2e-6
    assert np.array_equal(idx[~near], ref_idx[~near])
    # the packed bytes are the packed indices
    packed, n2, s2 = oracle.tq3_encode(x, bits)
    assert np.array_equal(packed, oracle.tq3_pack(idx))
    assert np.array_equal(n2, norms) and np.array_equal(s2, scales)


def test_tq3_decode_matches_dense_float64(oracle):
    bits = inputs.tq3_sign_bits()
    signs = oracle.tq3_signs(bits).astype(np.float64)
    c, _ = oracle.tq3_tables()
    idx = inputs.uniform_int((32, 128), 8, seed=22)
    packed = oracle.tq3_pack(idx)
    norms = (np.abs(inputs.gaussian((32,), seed=23)) * 5 + 0.5).astype(np.float32)
    scales = (np.abs(inputs.gaussian((32,), seed=24)) * 0.3 + 0.05).astype(np.float32)
    out = oracle.tq3_decode(packed, norms, scales, bits)
    H = oracle.hadamard_dense(128).astype(np.float64)
    v = c[idx].astype(np.float64) * scales[:, None]
    ref = (v @ H.T / math.sqrt(128)) * signs * norms[:, None]
    rel = np.abs(out - ref).max(axis=1) / np.abs(ref).max(axis=1)
    assert rel.max() < 2e-6
    out16 = oracle.tq3_decode(packed, norms, scales, bits, out_bf16=True)
    assert np.array_equal(out16, oracle.f32_array_to_bf16(out))


def test_tq3_zero_vector(oracle):
    bits = inputs.tq3_sign_bits()
    packed, n, s = oracle.tq3_encode(np.zeros((2, 128), np.float32), bits)
    assert np.all(n == np.float32(1e-8)) and np.all(s == np.float32(1e-8))
    assert packed.tobytes() == bytes.fromhex("dbb66d") * 32
    out = oracle.tq3_decode(packed, n, s, bits)
    assert np.abs(out).max() < 1e-15


def _post_flip_roundtrip(oracle, x, signs):
    """The pre-fix ordering the commit message describes: FWHT first, sign flips afterwards,
    composed from the oracle's own primitives (normalise, butterfly, bucketize, pack)."""
    c, _ = oracle.tq3_tables()
    out = []
    for row in x:
        n = np.float32(max(np.float32(math.sqrt(float(np.sum(row.astype(np.float64) ** 2)))), np.float32(1e-8)))
        xh = oracle.fwht((row / n).astype(np.float32)) * signs
        s = np.float32(max(np.abs(xh).max(), np.float32(1e-8)))
        idx = np.array([oracle.tq3_bucketize(v) for v in (xh / s).astype(np.float32)], np.uint8)
        idx = oracle.tq3_unpack(oracle.tq3_pack(idx))[0]
        y = oracle.fwht((c[idx] * s * signs).astype(np.float32)) * n
        out.append(y)
    return np.array(out, np.float32)


def test_constant_block_closed_form_without_preflips(oracle):
    """Without pre-transform flips a constant block collapses onto Hadamard coefficient 0: index
    7 there and index 3 everywhere else. Closed form: cos = c7 / sqrt(c7^2 + 127 c3^2),
    rel-L2 = sqrt((1 - c7)^2 + 127 c3^2); the commit message prints 0.611 and 1.27."""
    g = golden_dict("page_numbers.txt")
    c, _ = oracle.tq3_tables()
    c7, c3 = float(c[7]), float(c[3])
    cos_cf = c7 / math.sqrt(c7 ** 2 + 127 * c3 ** 2)
    rel_cf = math.sqrt((1 - c7) ** 2 + 127 * c3 ** 2)
    assert round(cos_cf, 3) == float(g["post_flip_constant_cosine"][0])
    assert round(rel_cf, 2) == float(g["post_flip_constant_rel_l2"][0])
    ones = np.ones(128, np.uint8)  # all draws 1 = no flips
    for val in (1.0, 2.5):
        x = np.full((1, 128), val, np.float32)
        xs, idx, _, _ = oracle.tq3_encode_debug(x, ones)
        assert idx[0, 0] == 7 and np.all(idx[0, 1:] == 3)
        p, n, s = oracle.tq3_encode(x, ones)
        xr = oracle.tq3_decode(p, n, s, ones)[0].astype(np.float64)
        cos = xr.sum() / (np.linalg.norm(xr) * math.sqrt(128))
        rel = np.linalg.norm(xr - val) / (val * math.sqrt(128))
        assert abs(cos - cos_cf) < 1e-5 and abs(rel - rel_cf) < 1e-5


def test_post_transform_flips_are_a_noop_and_preflips_rescue(oracle):
    """Commit message of "tq3_core.py": flips after the transform give a bit-identical
    reconstruction; flips before it spread a constant block (cos > 0.97)."""
    bits = inputs.tq3_sign_bits()
    signs = oracle.tq3_signs(bits)
    ones = np.ones(128, np.uint8)
    x = np.concatenate([inputs.gaussian((6, 128), seed=31), np.full((1, 128), 2.5, np.float32)])
    post = _post_flip_roundtrip(oracle, x, signs)
    noflip = oracle.tq3_decode(*oracle.tq3_encode(x, ones), ones)
    xs, _, _, _ = oracle.tq3_encode_debug(x, ones)
    no_zero = ~np.any(xs == 0, axis=1)
    assert no_zero[:6].all()
    assert np.array_equal(post[no_zero], noflip[no_zero])
    # with the seed-42 pre-flips the constant block has exactly 11 zero coefficients (an exact
    # 0.0 boundary tie each) and comes back at cosine ~0.983
    const = np.full((1, 128), 2.5, np.float32)
    xs, idx, _, _ = oracle.tq3_encode_debug(const, bits)
    assert int(np.sum(xs == 0)) == 11 and np.all(idx[xs == 0] == 3)
    xr = oracle.tq3_decode(*oracle.tq3_encode(const, bits), bits)[0].astype(np.float64)
    cos = xr.sum() / (np.linalg.norm(xr) * math.sqrt(128))
    assert cos > 0.97 and abs(cos - 0.98285) < 1e-4


def test_tq3_gaussian_roundtrip_cosine(oracle):
    """Page self_test tests 1-2: mean cosine over Gaussian vectors above 0.97."""
    bits = inputs.tq3_sign_bits()
    x = inputs.tq3_roundtrip()
    p, n, s = oracle.tq3_encode(x, bits)
    xr = oracle.tq3_decode(p, n, s, bits).astype(np.float64)
    x64 = x.astype(np.float64)
    cos = (x64 * xr).sum(1) / (np.linalg.norm(x64, axis=1) * np.linalg.norm(xr, axis=1))
    assert cos[:4064].mean() > 0.97
    assert 0.94 < cos[:4064].min() < 0.97
    assert np.all(cos[4064:] > 0.97)


def test_tq3_bf16_input_is_exact_widening(oracle):
    bits = inputs.tq3_sign_bits()
    xb = inputs.to_bf16_bits(torch.from_numpy(inputs.gaussian((16, 128), seed=41)))
    a = oracle.tq3_encode(xb, bits, is_bf16=True)
    b = oracle.tq3_encode(oracle.bf16_array_to_f32(xb), bits)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_bf16_rounding_matches_torch(oracle):
    x = np.concatenate([inputs.gaussian((20000,), seed=51) * 100,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, -0.0], np.float32)])
    x = x.astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16(v) for v in x[:2000]] + list(oracle.f32_array_to_bf16(x[2000:])), np.uint16)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------------------------------------
# Lloyd-Max ("orbit_quant.py" gaussian_lloyd_max)
# ------------------------------------------------------------------------------------------
def test_erfinv_inverts_erf(oracle):
    for t in (-0.999, -0.5, -0.1, 0.0, 0.3, 0.5, 0.9, 0.99999):
        y = oracle.erfinv(t)
        assert abs(math.erf(y) - t) < 4e-16
    assert abs(oracle.erfinv(0.5) - 0.4769362762044699) < 1e-15


def test_lloyd_max_textbook_levels(oracle):
    for parts in read_golden("lloyd_max_max1960.txt"):
        bits = int(parts[0])
        table = np.array([float(v) for v in parts[1:]])
        c = oracle.gaussian_lloyd_max(bits).astype(np.float64)
        half = c[len(c) // 2:]
        # Max's table is good to about 1e-4 (it is a 1960 hand/numeric computation printed to 4
        # decimals); the 4-bit iteration is not converged after the page's 200 steps
        tol = 1e-3 if bits == 4 else 1e-4
        assert np.abs(half - table).max() < tol, (bits, half, table)
        assert np.array_equal(c, -c[::-1])


def test_lloyd_max_fixed_point_by_quadrature(oracle):
    """Centroid condition checked with numerical integration (not the update formula): each level
    is the conditional mean of N(0,1) on its cell between the midpoint edges."""
    from scipy import integrate
    phi = lambda t: math.exp(-t * t / 2) / math.sqrt(2 * math.pi)
    for bits, tol in ((2, 1e-9), (3, 1e-9), (4, 1e-4)):
        c = oracle.gaussian_lloyd_max_f64(bits)
        e = np.concatenate([[-np.inf], (c[:-1] + c[1:]) / 2, [np.inf]])
        for k in range(len(c)):
            lo, hi = max(e[k], -12.0), min(e[k + 1], 12.0)
            m1 = integrate.quad(lambda t: t * phi(t), lo, hi, epsabs=1e-14, epsrel=1e-12)[0]
            m0 = integrate.quad(phi, lo, hi, epsabs=1e-14, epsrel=1e-12)[0]
            assert abs(m1 / m0 - c[k]) < tol, (bits, k, m1 / m0, c[k])


def test_lloyd_max_fp32_bits_exact(oracle):
    """The fp32 codebooks of gaussian_lloyd_max(bits, iters=200), bit for bit, against values
    computed by an independent float64 implementation of the page's iteration. At 4 bits the
    iterate still moves by about 1.8e-5 per step, so 199 or 201 iterations must differ in every
    level: this catches an off-by-one iteration count that the 1e-3 / 1e-4 checks above allow."""
    seen = set()
    for parts in read_golden("lloyd_max_fp32.txt"):
        bits = int(parts[0])
        want = np.array([int(v, 16) for v in parts[1:]], dtype=np.uint32)
        assert want.size == 1 << bits
        got = oracle.gaussian_lloyd_max(bits).view(np.uint32)
        assert np.array_equal(got, want), (bits, [f"{v:08x}" for v in got])
        seen.add(bits)
    assert seen == {2, 3, 4}
    c200 = oracle.gaussian_lloyd_max(4, 200)
    for iters in (199, 201):
        other = oracle.gaussian_lloyd_max(4, iters)
        assert np.all(other != c200), iters
        assert np.abs(other.astype(np.float64) - c200).max() < 5e-5
    for bits in (2, 3):  # fp32 fixed points: one more or one fewer step changes nothing
        assert np.array_equal(oracle.gaussian_lloyd_max(bits, 199), oracle.gaussian_lloyd_max(bits, 200))
        assert np.array_equal(oracle.gaussian_lloyd_max(bits, 201), oracle.gaussian_lloyd_max(bits, 200))


def test_rpbh_codebook_scaling(oracle):
    for bits in (2, 3, 4):
        for d in (3072, 11008):
            cb = oracle.rpbh_codebook(bits, d)
            ref = oracle.gaussian_lloyd_max(bits) * np.float32(d ** -0.5)
            assert np.array_equal(cb, ref)
            assert np.array_equal(cb, -cb[::-1])


# ------------------------------------------------------------------------------------------
# RPBH ("orbit_quant.py" rpbh_forward / rpbh_inverse / _quantize_rows / _dequantize_rotated)
# ------------------------------------------------------------------------------------------
def _dense_rotation(oracle, d, perm, signs):
    """blkdiag(H_h) D P as a float64 matrix, built from its definition."""
    h = d & -d
    H = oracle.hadamard_dense(h).astype(np.float64) / math.sqrt(h)
    B = np.kron(np.eye(d // h), H)
    P = np.zeros((d, d))
    P[np.arange(d), perm] = 1.0
    return B @ np.diag(signs.astype(np.float64)) @ P


def test_hadamard_block_size(oracle):
    for d, h in ((11008, 256), (3072, 1024), (96, 32), (4096, 4096), (100, 4), (7, 1)):
        assert oracle.hadamard_block_size(d) == h


@pytest.mark.parametrize("d", [32, 96, 192, 640])
def test_rpbh_forward_equals_dense_rotation(oracle, d):
    perm, signs = inputs.rpbh_params(d)
    h = d & -d
    R = _dense_rotation(oracle, d, perm, signs)
    assert np.allclose(R @ R.T, np.eye(d), atol=1e-12)
    x = inputs.gaussian((5, d), seed=d)
    y = oracle.rpbh_forward(x, perm, signs, h)
    assert np.abs(y - x.astype(np.float64) @ R.T).max() < 1e-5
    inv = np.argsort(perm).astype(np.int32)
    z = oracle.rpbh_inverse(y, inv, signs, h)
    assert np.abs(z - x).max() < 1e-5
    # (W P^T)(P x) = W x: the rotations cancel in a matmul
    W = inputs.gaussian((7, d), seed=d + 1)
    Wr = oracle.rpbh_forward(W, perm, signs, h)
    assert np.allclose(Wr.astype(np.float64) @ y.astype(np.float64).T,
                       W.astype(np.float64) @ x.astype(np.float64).T, atol=1e-3)


def test_rpbh_params_tables():
    perm, signs = inputs.rpbh_params(11008)
    assert perm[:8].tolist() == [5354, 4279, 699, 7415, 6590, 9455, 7865, 10634]
    assert signs[:8].tolist() == [-1, 1, 1, 1, 1, -1, -1, 1]
    perm, signs = inputs.rpbh_params(3072)
    assert perm[:8].tolist() == [1335, 2402, 236, 2484, 1736, 740, 2957, 92]
    assert signs[:8].tolist() == [1, 1, 1, 1, -1, 1, 1, 1]
    assert np.array_equal(np.sort(perm), np.arange(3072))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_rpbh_quantize_matches_dense_and_brute_force(oracle, bits):
    d, rows = 192, 12
    perm, signs = inputs.rpbh_params(d)
    h = d & -d
    cb = oracle.rpbh_codebook(bits, d)
    w = inputs.gaussian((rows, d), seed=60 + bits) * 0.02
    w[3] = 0.0  # a zero row
    packed, norms, codes, unit = oracle.rpbh_quantize(w, perm, signs, h, cb, bits, want_debug=True)
    R = _dense_rotation(oracle, d, perm, signs)
    wr = w.astype(np.float64) @ R.T
    rho = np.linalg.norm(wr, axis=1)
    assert np.allclose(norms, rho, rtol=1e-6, atol=0)
    assert norms[3] == 0 and np.all(codes[3] == (1 << bits) // 2 - 1)
    u = wr / (rho[:, None] + 1e-10)
    assert np.abs(unit - u).max() < 1e-6
    edges = (cb[:-1].astype(np.float64) + cb[1:]) / 2
    near = np.min(np.abs(u[..., None] - edges), axis=-1) * math.sqrt(d) < 1e-5
    bf = np.array([[oracle.nearest_centroid(v, cb) for v in row] for row in unit])
    assert np.array_equal(bf, codes)  # brute-force nearest centroid on the same fp32 values
    ref = np.searchsorted(edges, u, side="left")
    assert np.array_equal(codes[~near], ref[~near])
    assert np.array_equal(packed, oracle.pack_codes(codes, bits))


def test_rpbh_dequantize_matches_dense(oracle):
    d, rows, bits = 96, 6, 3
    perm, signs = inputs.rpbh_params(d)
    h = d & -d
    cb = oracle.rpbh_codebook(bits, d)
    codes = inputs.uniform_int((rows, d), 8, seed=70)
    packed = oracle.pack_codes(codes, bits)
    norms = (np.abs(inputs.gaussian((rows,), seed=71)) + 0.1).astype(np.float32)
    wrot = oracle.rpbh_dequantize_rotated(packed, norms, rows, d, bits, cb)
    assert np.array_equal(wrot, cb[codes] * norms[:, None])
    w16 = oracle.rpbh_dequantize_rotated(packed, norms, rows, d, bits, cb, out_bf16=True)
    ref16 = (torch.from_numpy(cb).to(torch.bfloat16)[torch.from_numpy(codes.astype(np.int64))] *
             torch.from_numpy(norms).to(torch.bfloat16)[:, None])
    assert np.array_equal(w16, ref16.view(torch.int16).numpy().view(np.uint16))
    inv = np.argsort(perm).astype(np.int32)
    w = oracle.rpbh_dequantize(packed, norms, rows, d, bits, cb, inv, signs, h)
    R = _dense_rotation(oracle, d, perm, signs)
    assert np.abs(w - wrot.astype(np.float64) @ R).max() < 1e-5


def test_tq3_records_are_the_pages_56_bytes(oracle):
    """A record is the page's compressed size per vector (tq3_memory_bytes: 56 bytes), laid out as
    the 48 packed bytes, then the norm and the scale as little-endian fp32; the split is exact."""
    import struct
    comp, _, _ = oracle.tq3_memory_bytes((3, 128))
    x = inputs.gaussian((3, 128), seed=75).astype(np.float32)
    p, n, sc = oracle.tq3_encode(x, inputs.tq3_sign_bits())
    r = oracle.tq3_to_records(p, n, sc)
    assert r.shape == (3, 56) and r.size == comp
    for v in range(3):
        assert bytes(r[v, :48]) == bytes(p[v])
        assert bytes(r[v, 48:]) == struct.pack('<ff', float(n[v]), float(sc[v]))
    p2, n2, s2 = oracle.tq3_from_records(r)
    assert np.array_equal(p2, p) and np.array_equal(n2, n) and np.array_equal(s2, sc)


def test_rpbh_linear_one_hot_and_zero_inputs(oracle):
    """forward's F.linear on the rotated activations: a one-hot activation row e_k returns column k
    of the bf16 rotated weight plus the bias (so the product is x W'^T, not a transpose of it), and
    zero activations return the bias exactly."""
    out_f, d, bits = 5, 64, 3
    cb = oracle.rpbh_codebook(bits, d)
    codes = inputs.uniform_int((out_f, d), 8, seed=72)
    packed = oracle.pack_codes(codes, bits)
    norms = (np.abs(inputs.gaussian((out_f,), seed=73)) + 0.1).astype(np.float32)
    bias = oracle.f32_array_to_bf16(inputs.gaussian((out_f,), seed=74).astype(np.float32))
    one = oracle.f32_array_to_bf16(np.eye(d, dtype=np.float32))
    y, a = oracle.rpbh_linear(packed, norms, out_f, d, bits, cb, one, bias)
    w16 = oracle.bf16_array_to_f32(oracle.rpbh_dequantize_rotated(packed, norms, out_f, d, bits, cb, out_bf16=True))
    b32 = oracle.bf16_array_to_f32(bias)
    assert y.shape == (d, out_f)
    assert np.array_equal(y, w16.T.astype(np.float64) + b32[None, :].astype(np.float64))
    assert np.array_equal(a, np.abs(w16.T).astype(np.float64))
    zero = np.zeros((3, d), np.uint16)
    y0, a0 = oracle.rpbh_linear(packed, norms, out_f, d, bits, cb, zero, bias)
    assert np.array_equal(y0, np.broadcast_to(b32.astype(np.float64), (3, out_f)))
    assert not a0.any()


def test_rpbh_rotate_bf16_matches_dense(oracle):
    d = 640
    perm, signs = inputs.rpbh_params(d)
    h = d & -d
    xb = inputs.activations(4, d, seed=80)
    out = oracle.rpbh_rotate_bf16(xb, perm, signs, h)
    R = _dense_rotation(oracle, d, perm, signs)
    ref = oracle.bf16_array_to_f32(xb).astype(np.float64) @ R.T
    got = oracle.bf16_array_to_f32(out).astype(np.float64)
    # one bf16 rounding of a value that is itself within 1e-6 of the float64 result
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2 ** -8 + 1e-6)


def _attn_cache(oracle, heads, S, seed, same_keys=False):
    bits = inputs.tq3_sign_bits()
    x = inputs.gaussian((2, heads, S, 128), seed=seed).astype(np.float32)
    if same_keys:
        x[:, :, :, :] = x[:, :, :1, :]
    recs = [oracle.tq3_to_records(*oracle.tq3_encode(x[i].reshape(-1, 128), bits)).reshape(heads, S, 56)
            for i in range(2)]
    dec = [oracle.tq3_decode(*oracle.tq3_from_records(r.reshape(-1, 56)), bits).reshape(heads, S, 128)
           .astype(np.float64) for r in recs]
    return bits, recs[0], recs[1], dec[0], dec[1]


def test_tq3_attention_closed_forms(oracle):
    """Attention over the decoded cache: one key returns its value; identical keys return their
    value whatever the query; a zero query averages the values; permuting the keys together with
    their values changes nothing."""
    bits, kr, vr, k, v = _attn_cache(oracle, 2, 1, seed=80)
    q = inputs.gaussian((2, 3, 128), seed=81).astype(np.float32)
    assert np.allclose(oracle.tq3_attention(q, kr, vr, bits, 0.088), np.repeat(v, 3, axis=1), rtol=0, atol=1e-12)

    bits, kr, vr, k, v = _attn_cache(oracle, 1, 9, seed=82, same_keys=True)
    out = oracle.tq3_attention(q[:1], kr, vr, bits, 0.5)
    assert np.allclose(out, np.repeat(v[:, :1], 3, axis=1), rtol=0, atol=1e-12)

    bits, kr, vr, k, v = _attn_cache(oracle, 2, 17, seed=83)
    out = oracle.tq3_attention(np.zeros((2, 2, 128), np.float32), kr, vr, bits, 0.3)
    assert np.allclose(out, np.repeat(v.mean(axis=1, keepdims=True), 2, axis=1), rtol=0, atol=1e-12)

    q = inputs.gaussian((2, 4, 128), seed=84).astype(np.float32)
    perm = np.random.default_rng(0).permutation(17)
    a = oracle.tq3_attention(q, kr, vr, bits, 0.1)
    b = oracle.tq3_attention(q, kr[:, perm], vr[:, perm], bits, 0.1)
    assert np.allclose(a, b, rtol=0, atol=1e-12)


def test_tq3_attention_hard_max_picks_the_value_of_the_best_key(oracle):
    """With a large softmax scale the weights collapse onto the key with the largest q . k: the
    output is that key's value (not its key, and not the value of the smallest q . k)."""
    bits, kr, vr, k, v = _attn_cache(oracle, 1, 12, seed=85)
    q = inputs.gaussian((1, 2, 128), seed=86).astype(np.float32)
    out = oracle.tq3_attention(q, kr, vr, bits, 1e4)
    for r in range(2):
        best = int(np.argmax(k[0] @ q[0, r].astype(np.float64)))
        assert np.allclose(out[0, r], v[0, best], rtol=0, atol=1e-9)


def test_tq3_dot_products_in_the_indices_basis(oracle):
    """The decoded vector is k = s . H(c[idx] scale) post norm with H the symmetric Sylvester matrix,
    so q . k = norm scale post (H (s . q)) . c[idx] and sum_j w_j k_j = s . H(sum_j w_j norm_j scale_j
    c[idx_j]) post: attention can score and sum without decoding. Checked in fp64 against the
    oracle's decoded fp32 vectors (agreement to fp32 rounding)."""
    bits = inputs.tq3_sign_bits()
    x = inputs.gaussian((40, 128), seed=88).astype(np.float32)
    p, n, sc = oracle.tq3_encode(x, bits)
    k = oracle.tq3_decode(p, n, sc, bits).astype(np.float64)
    c, _ = oracle.tq3_tables()
    cv = c[oracle.tq3_unpack(p)].astype(np.float64)                       # [40, 128] centroids
    s = oracle.tq3_signs(bits).astype(np.float64)
    H = oracle.hadamard_dense(128).astype(np.float64)
    post = float(np.float32(1.0 / np.sqrt(128.0)))
    coef = n.astype(np.float64) * sc.astype(np.float64) * post
    q = inputs.gaussian((3, 128), seed=89).astype(np.float64)
    direct = q @ k.T
    rotated = ((H @ (s * q).T).T @ cv.T) * coef[None, :]
    assert np.abs(direct - rotated).max() <= 1e-5 * np.abs(q).sum(axis=1).max() * np.abs(k).max()
    w = inputs.gaussian((40,), seed=90).astype(np.float64)
    direct_v = w @ k
    rotated_v = s * (H @ ((w * coef) @ cv))
    assert np.abs(direct_v - rotated_v).max() <= 1e-5 * np.abs(w).sum() * np.abs(k).max()


def test_tq3_tie_counts_of_the_round_trip_workload(oracle):
    """The stored oracle counts for the 4096-vector round trip (tests/golden/tq3_tie_counts.txt)
    still hold: 352 exact zeros, all from the 32 constant blocks (11 each, the pre-flip pin above),
    inside 649 coefficients within 1e-6 of a boundary."""
    from weight_quantization_b200 import inputs
    want = {r[0]: tuple(int(v) for v in r[1:]) for r in read_golden("tq3_tie_counts.txt")}
    x = inputs.tq3_roundtrip()
    xs, _, _, _ = oracle.tq3_encode_debug(x, inputs.tq3_sign_bits())
    _, B = oracle.tq3_tables()
    near = np.zeros(xs.shape, bool)
    for b in B.astype(np.float64):
        near |= np.abs(xs.astype(np.float64) - b) < 1e-6
    assert (xs.shape[0], int(near.sum()), int((xs == 0).sum())) == want["tq3_roundtrip_fp32"]
    assert int((xs[4064:] == 0).sum()) == 32 * 11 == want["tq3_roundtrip_fp32"][2]
