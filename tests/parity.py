"""Comparison rules between the CUDA library and the oracle.

Rules (the contract these tests enforce):
* packed bytes are bit-exact, except TQ3 coefficients whose oracle value xs lies within 1e-6 of a
  codebook boundary and RPBH coefficients whose oracle unit value u lies within 1e-6 of an edge
  when measured in N(0,1) units (|u - e| * sqrt(d) < 1e-6); each such coefficient is counted;
* norms and scales within 1e-5 relative;
* fp32 reconstructions within 1e-5 relative per vector/row (max|diff| / max|oracle|);
* bf16 outputs within 1e-2 relative per vector/row.
"""
import math

import numpy as np

TIE_WINDOW = 1e-6
NORM_RTOL = 1e-5
F32_RTOL = 1e-5
BF16_RTOL = 1e-2


def rel_rows(got, ref):
    got = np.asarray(got, np.float64).reshape(ref.shape[0], -1)
    ref = np.asarray(ref, np.float64).reshape(ref.shape[0], -1)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return np.abs(got - ref).max(axis=1) / den


def check_tq3_encode(oracle, x, sign_bits, is_bf16, g_packed, g_norms, g_scales, ref=None):
    """Compare GPU encode outputs with the oracle. Returns a dict of counts.

    ref: the oracle's tq3_encode_debug(x, sign_bits, is_bf16) result, when the caller has it.
    """
    xs, idx, n, s = ref if ref is not None else oracle.tq3_encode_debug(x, sign_bits, is_bf16=is_bf16)
    g_packed = np.asarray(g_packed).reshape(-1, 48)
    g_idx = oracle.tq3_unpack(g_packed)
    _, B = oracle.tq3_tables()
    mism = g_idx != idx
    n_mism = int(mism.sum())
    if n_mism:
        dist = np.min(np.abs(xs[mism][:, None].astype(np.float64) - B.astype(np.float64)), axis=1)
        assert np.all(dist < TIE_WINDOW), f"index mismatch outside the tie window: max dist {dist.max()}"
        assert np.all(np.abs(g_idx[mism].astype(int) - idx[mism].astype(int)) == 1)
    rows_ok = ~mism.any(axis=1)
    ref_packed = oracle.tq3_pack(idx)
    assert np.array_equal(g_packed[rows_ok], ref_packed[rows_ok])
    g_norms = np.asarray(g_norms, np.float32).reshape(-1)
    g_scales = np.asarray(g_scales, np.float32).reshape(-1)
    # a norm beyond the fp32 range is +inf on the page (torch.norm in fp32): it must be +inf here too
    fin = np.isfinite(n)
    assert np.array_equal(g_norms[~fin], n[~fin]), "norms that overflow fp32 must be +inf"
    rn = np.abs(g_norms[fin].astype(np.float64) - n[fin]) / np.abs(n[fin])
    rs = np.abs(g_scales.astype(np.float64) - s) / np.abs(s)
    assert rn.size == 0 or rn.max() <= NORM_RTOL, rn.max()
    assert rs.max() <= NORM_RTOL, rs.max()
    near = np.zeros(xs.shape, bool)
    for b in B.astype(np.float64):
        near |= np.abs(xs.astype(np.float64) - b) < TIE_WINDOW
    far = 0
    if n_mism:
        far = int((dist >= 1e-7).sum())
    return {
        "vectors": int(idx.shape[0]),
        "index_mismatches": n_mism,
        "mismatches_beyond_1e-7": far,
        "coeffs_in_tie_window": int(near.sum()),
        "exact_zero_coeffs": int((xs == 0).sum()),
        "bytes_equal": bool(np.array_equal(g_packed, ref_packed)),
        "norms_equal": int((g_norms == n).sum()),
        "scales_equal": int((g_scales == s).sum()),
    }


def check_tq3_decode(oracle, packed, norms, scales, sign_bits, g_out, out_bf16):
    ref = oracle.tq3_decode(packed, norms, scales, sign_bits, out_bf16=out_bf16)
    g_out = np.asarray(g_out).reshape(ref.shape)
    if out_bf16:
        r = rel_rows(oracle.bf16_array_to_f32(g_out), oracle.bf16_array_to_f32(ref))
        assert r.max() <= BF16_RTOL, r.max()
    else:
        r = rel_rows(g_out, ref)
        assert r.max() <= F32_RTOL, r.max()
    return {"vectors": int(ref.shape[0]), "max_rel": float(r.max()),
            "bit_exact": bool(np.array_equal(g_out.view(np.uint8), ref.view(np.uint8)))}


def check_rpbh_quantize(oracle, w, is_bf16, perm, signs, h, cb, bits, g_packed):
    """Compare GPU packed codes with the oracle; returns (stats, oracle packed, oracle fp32 norms)."""
    rows, d = w.shape
    packed, norms, codes, unit = oracle.rpbh_quantize(w, perm, signs, h, cb, bits, is_bf16=is_bf16,
                                                      want_debug=True)
    g_packed = np.asarray(g_packed)
    g_codes = oracle.unpack_codes(g_packed, bits, rows * d).reshape(rows, d)
    mism = g_codes != codes
    n_mism = int(mism.sum())
    edges = (cb[:-1] + cb[1:]) / np.float32(2)
    if n_mism:
        dist = np.min(np.abs(unit[mism][:, None].astype(np.float64) - edges.astype(np.float64)), axis=1)
        assert np.all(dist * math.sqrt(d) < TIE_WINDOW), f"code mismatch outside the tie window {dist.max()}"
    bytes_equal = bool(np.array_equal(g_packed, packed))
    if n_mism == 0:
        assert bytes_equal
    return {"rows": rows, "code_mismatches": n_mism, "bytes_equal": bytes_equal}, packed, norms


def check_norms(got_f32, ref_f32):
    got = np.asarray(got_f32, np.float64)
    ref = np.asarray(ref_f32, np.float64)
    rn = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
    assert rn.max() <= NORM_RTOL, rn.max()
    return int((got == ref).sum())
