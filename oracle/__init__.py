"""ctypes front end of the C99 oracle (TEST INFRASTRUCTURE ONLY).

The oracle restates, step by step and in fp32 where the pages compute in fp32, what the pages
"tq3_core.py" (TQ3 KV codec) and "orbit_quant.py" (OrbitQuant RPBH weights) compute. Only the
tests, the smoke check and the benchmark's CPU-baseline leg use it; the CUDA library never does.
All arrays are numpy; bf16 data travels as raw uint16 bit patterns.
"""
from __future__ import annotations

import ctypes as C
import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(_build.build())
        _declare(_lib)
    return _lib


def _p(a):
    return a.ctypes.data_as(C.c_void_p)


def _declare(L):
    vp, i64, i32, f32 = C.c_void_p, C.c_int64, C.c_int, C.c_float
    sig = {
        "or_bf16_to_f32": (f32, [C.c_uint16]),
        "or_f32_to_bf16": (C.c_uint16, [f32]),
        "or_fwht": (None, [vp, i64, f32]),
        "or_tq3_fwht_post": (f32, [i64]),
        "or_rpbh_fwht_post": (f32, [i64]),
        "or_tq3_encode": (None, [vp, i32, i64, vp, vp, vp, vp]),
        "or_tq3_encode_debug": (None, [vp, i32, i64, vp, vp, vp, vp, vp]),
        "or_tq3_decode": (None, [vp, vp, vp, i64, vp, vp, i32]),
        "or_tq3_bucketize": (C.c_uint8, [f32]),
        "or_tq3_pack": (None, [vp, i64, vp]),
        "or_tq3_unpack": (None, [vp, i64, vp]),
        "or_tq3_memory_bytes": (i64, [vp, i32, vp]),
        "or_tq3_tables": (None, [vp, vp]),
        "or_erfinv": (C.c_double, [C.c_double]),
        "or_gaussian_lloyd_max": (None, [i32, i32, vp]),
        "or_gaussian_lloyd_max_f64": (None, [i32, i32, vp]),
        "or_hadamard_block_size": (i64, [i64]),
        "or_rpbh_codebook": (None, [i32, i64, vp]),
        "or_rpbh_forward": (None, [vp, i64, i64, vp, vp, i64, vp]),
        "or_rpbh_inverse": (None, [vp, i64, i64, vp, vp, i64, vp]),
        "or_packed_bytes": (i64, [i64, i32]),
        "or_pack_codes": (None, [vp, i64, i32, vp]),
        "or_unpack_codes": (None, [vp, i64, i32, vp]),
        "or_rpbh_quantize": (None, [vp, i32, i64, i64, vp, vp, i64, vp, i32, vp, vp, vp, vp]),
        "or_rpbh_dequantize_rotated": (None, [vp, vp, i64, i64, i32, vp, vp, i32]),
        "or_rpbh_dequantize": (None, [vp, vp, i64, i64, i32, vp, vp, vp, i64, vp]),
        "or_rpbh_rotate_bf16": (None, [vp, i64, i64, vp, vp, i64, vp]),
        "or_hadamard_dense": (None, [i64, vp]),
        "or_nearest_centroid": (i32, [f32, vp, i32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------------------------------------
# TQ3 (page "tq3_core.py")
# ---------------------------------------------------------------------------------------------
def tq3_signs(bits) -> np.ndarray:
    """_generate_sign_flips: the drawn bits mapped to +-1.0 (bits * 2.0 - 1.0)."""
    return np.asarray(bits, dtype=np.float32) * np.float32(2.0) - np.float32(1.0)


def tq3_tables():
    c = np.zeros(8, np.float32)
    b = np.zeros(7, np.float32)
    lib().or_tq3_tables(_p(c), _p(b))
    return c, b


def tq3_encode(x, sign_bits, is_bf16: bool = False):
    """tq3_quantize on [n_vec, 128] rows (fp32, or uint16 bf16 bits with is_bf16=True)."""
    x = _c(x, np.uint16 if is_bf16 else np.float32).reshape(-1, 128)
    n = x.shape[0]
    signs = tq3_signs(sign_bits)
    packed = np.zeros((n, 48), np.uint8)
    norms = np.zeros(n, np.float32)
    scales = np.zeros(n, np.float32)
    lib().or_tq3_encode(_p(x), int(is_bf16), n, _p(signs), _p(packed), _p(norms), _p(scales))
    return packed, norms, scales


def tq3_encode_debug(x, sign_bits, is_bf16: bool = False):
    """Like tq3_encode but returns (xs, idx, norms, scales) before packing."""
    x = _c(x, np.uint16 if is_bf16 else np.float32).reshape(-1, 128)
    n = x.shape[0]
    signs = tq3_signs(sign_bits)
    xs = np.zeros((n, 128), np.float32)
    idx = np.zeros((n, 128), np.uint8)
    norms = np.zeros(n, np.float32)
    scales = np.zeros(n, np.float32)
    lib().or_tq3_encode_debug(_p(x), int(is_bf16), n, _p(signs), _p(xs), _p(idx), _p(norms), _p(scales))
    return xs, idx, norms, scales


def tq3_decode(packed, norms, scales, sign_bits, out_bf16: bool = False):
    """tq3_dequantize; fp32 out, or bf16 bits rounded once from the fp32 result."""
    packed = _c(packed, np.uint8).reshape(-1, 48)
    n = packed.shape[0]
    norms = _c(norms, np.float32)
    scales = _c(scales, np.float32)
    signs = tq3_signs(sign_bits)
    out = np.zeros((n, 128), np.uint16 if out_bf16 else np.float32)
    lib().or_tq3_decode(_p(packed), _p(norms), _p(scales), n, _p(signs), _p(out), int(out_bf16))
    return out


def tq3_bucketize(v: float) -> int:
    return int(lib().or_tq3_bucketize(float(v)))


def tq3_pack(idx):
    idx = _c(idx, np.uint8).reshape(-1, 128)
    out = np.zeros((idx.shape[0], 48), np.uint8)
    lib().or_tq3_pack(_p(idx), idx.shape[0], _p(out))
    return out


def tq3_unpack(packed):
    packed = _c(packed, np.uint8).reshape(-1, 48)
    out = np.zeros((packed.shape[0], 128), np.uint8)
    lib().or_tq3_unpack(_p(packed), packed.shape[0], _p(out))
    return out


def tq3_to_records(packed, norms, scales):
    """The 56-byte record of each vector ("56 bytes per vector", tq3_memory_bytes): its 48 packed bytes,
    then the fp32 norm and the fp32 scale, little-endian."""
    p = np.ascontiguousarray(packed, np.uint8).reshape(-1, 48)
    n = np.ascontiguousarray(norms, '<f4').reshape(-1, 1).view(np.uint8)
    s = np.ascontiguousarray(scales, '<f4').reshape(-1, 1).view(np.uint8)
    return np.concatenate([p, n, s], axis=1)


def tq3_attention(q, k_records, v_records, sign_bits, softmax_scale: float):
    """Scaled dot-product attention over a TQ3 K/V cache, by definition: every key and value is
    restored by tq3_dequantize (page "tq3_core.py", the page's own fp32 rounding), then, in fp64,
    out[h, r] = sum_j p_j v_j / sum_j p_j with p_j = exp(softmax_scale * q[h, r] . k_j - max_j).
    q [heads, m, 128] (fp32 values); k_records, v_records [heads, S, 56] records (tq3_to_records).
    Returns fp64 [heads, m, 128]."""
    q = np.asarray(q, np.float64)
    heads, m, _ = q.shape
    out = np.zeros((heads, m, 128), np.float64)
    for h in range(heads):
        k = tq3_decode(*tq3_from_records(k_records[h]), sign_bits).astype(np.float64)
        v = tq3_decode(*tq3_from_records(v_records[h]), sign_bits).astype(np.float64)
        logits = softmax_scale * (q[h] @ k.T)
        p = np.exp(logits - logits.max(axis=1, keepdims=True))
        out[h] = (p @ v) / p.sum(axis=1, keepdims=True)
    return out


def tq3_from_records(records):
    """The inverse of tq3_to_records: (packed [n, 48], norms [n], scales [n])."""
    r = np.ascontiguousarray(records, np.uint8).reshape(-1, 56)
    return (r[:, :48].copy(), r[:, 48:52].copy().view('<f4').reshape(-1).astype(np.float32),
            r[:, 52:56].copy().view('<f4').reshape(-1).astype(np.float32))


def tq3_memory_bytes(shape):
    s = np.asarray(shape, dtype=np.int64)
    orig = np.zeros(1, np.int64)
    comp = lib().or_tq3_memory_bytes(_p(s), len(shape), _p(orig))
    if comp < 0:
        raise ValueError(f"bad TQ3 shape {shape}")
    return int(comp), int(orig[0]), orig[0] / max(comp, 1)


def fwht(v, post=None):
    """Normalised FWHT of one power-of-two block (post defaults to fp32(1/sqrt(n)))."""
    v = _c(v, np.float32).copy()
    n = v.shape[0]
    if post is None:
        post = lib().or_tq3_fwht_post(n)
    lib().or_fwht(_p(v), n, float(post))
    return v


def bf16_to_f32(b) -> float:
    return float(lib().or_bf16_to_f32(int(b)))


def f32_to_bf16(f) -> int:
    return int(lib().or_f32_to_bf16(float(f)))


# ---------------------------------------------------------------------------------------------
# Lloyd-Max and RPBH (page "orbit_quant.py")
# ---------------------------------------------------------------------------------------------
def erfinv(t: float) -> float:
    return float(lib().or_erfinv(float(t)))


def gaussian_lloyd_max(bits: int, iters: int = 200) -> np.ndarray:
    out = np.zeros(1 << bits, np.float32)
    lib().or_gaussian_lloyd_max(bits, iters, _p(out))
    return out


def gaussian_lloyd_max_f64(bits: int, iters: int = 200) -> np.ndarray:
    out = np.zeros(1 << bits, np.float64)
    lib().or_gaussian_lloyd_max_f64(bits, iters, _p(out))
    return out


def hadamard_block_size(d: int) -> int:
    return int(lib().or_hadamard_block_size(d))


def rpbh_codebook(bits: int, d: int) -> np.ndarray:
    out = np.zeros(1 << bits, np.float32)
    lib().or_rpbh_codebook(bits, d, _p(out))
    return out


def rpbh_forward(x, perm, signs, h):
    x = _c(x, np.float32)
    rows, d = x.shape
    y = np.zeros_like(x)
    lib().or_rpbh_forward(_p(x), rows, d, _p(_c(perm, np.int32)), _p(_c(signs, np.int8)), h, _p(y))
    return y


def rpbh_inverse(y, inv_perm, signs, h):
    y = _c(y, np.float32)
    rows, d = y.shape
    out = np.zeros_like(y)
    lib().or_rpbh_inverse(_p(y), rows, d, _p(_c(inv_perm, np.int32)), _p(_c(signs, np.int8)), h, _p(out))
    return out


def packed_bytes(numel: int, bits: int) -> int:
    return int(lib().or_packed_bytes(numel, bits))


def pack_codes(codes, bits):
    codes = _c(codes, np.uint8).reshape(-1)
    out = np.zeros(packed_bytes(codes.size, bits), np.uint8)
    lib().or_pack_codes(_p(codes), codes.size, bits, _p(out))
    return out


def unpack_codes(packed, bits, numel):
    packed = _c(packed, np.uint8)
    out = np.zeros(numel, np.uint8)
    lib().or_unpack_codes(_p(packed), numel, bits, _p(out))
    return out


def rpbh_quantize(w, perm, signs, h, codebook, bits, is_bf16=False, want_debug=False):
    """_quantize_rows: returns (packed, fp32 row norms[, codes, unit])."""
    w = _c(w, np.uint16 if is_bf16 else np.float32)
    rows, d = w.shape
    packed = np.zeros(packed_bytes(rows * d, bits), np.uint8)
    norms = np.zeros(rows, np.float32)
    codes = np.zeros((rows, d), np.uint8) if want_debug else None
    unit = np.zeros((rows, d), np.float32) if want_debug else None
    lib().or_rpbh_quantize(_p(w), int(is_bf16), rows, d, _p(_c(perm, np.int32)), _p(_c(signs, np.int8)),
                           h, _p(_c(codebook, np.float32)), bits, _p(packed), _p(norms),
                           _p(codes) if want_debug else None, _p(unit) if want_debug else None)
    if want_debug:
        return packed, norms, codes, unit
    return packed, norms


def rpbh_dequantize_rotated(packed, row_norms_f32, rows, d, bits, codebook, out_bf16=False):
    out = np.zeros((rows, d), np.uint16 if out_bf16 else np.float32)
    lib().or_rpbh_dequantize_rotated(_p(_c(packed, np.uint8)), _p(_c(row_norms_f32, np.float32)), rows, d,
                                     bits, _p(_c(codebook, np.float32)), _p(out), int(out_bf16))
    return out


def rpbh_linear(packed, row_norms_f32, out_features, d, bits, codebook, x_rot_bits, bias_bits=None):
    """Page "orbit_quant.py", forward: F.linear(x_rot, W', bias) with W' the rotated-basis weight in
    bf16 (_dequantize_rotated in the weight dtype, as rpbh_dequantize_rotated(out_bf16=True)).
    The product is taken in fp64 (a library matmul). Returns (y, abs_sum): y [m, out_features] and
    abs_sum[i][n] = sum_k |x_rot[i][k] W'[n][k]|, which bounds the rounding of any fp32 evaluation."""
    wq = bf16_array_to_f32(rpbh_dequantize_rotated(packed, row_norms_f32, out_features, d, bits, codebook,
                                                   out_bf16=True)).astype(np.float64)
    x = bf16_array_to_f32(np.asarray(x_rot_bits, np.uint16)).astype(np.float64)
    y = x @ wq.T
    a = np.abs(x) @ np.abs(wq).T
    if bias_bits is not None:
        y = y + bf16_array_to_f32(np.asarray(bias_bits, np.uint16)).astype(np.float64)[None, :]
    return y, a


def rpbh_dequantize(packed, row_norms_f32, rows, d, bits, codebook, inv_perm, signs, h):
    out = np.zeros((rows, d), np.float32)
    lib().or_rpbh_dequantize(_p(_c(packed, np.uint8)), _p(_c(row_norms_f32, np.float32)), rows, d, bits,
                             _p(_c(codebook, np.float32)), _p(_c(inv_perm, np.int32)),
                             _p(_c(signs, np.int8)), h, _p(out))
    return out


def rpbh_rotate_bf16(x_bits, perm, signs, h):
    x = _c(x_bits, np.uint16)
    rows, d = x.shape
    out = np.zeros_like(x)
    lib().or_rpbh_rotate_bf16(_p(x), rows, d, _p(_c(perm, np.int32)), _p(_c(signs, np.int8)), h, _p(out))
    return out


def hadamard_dense(n: int) -> np.ndarray:
    H = np.zeros((n, n), np.int8)
    lib().or_hadamard_dense(n, _p(H))
    return H


def nearest_centroid(v: float, c) -> int:
    c = _c(c, np.float32)
    return int(lib().or_nearest_centroid(float(v), _p(c), c.size))


def bf16_array_to_f32(bits) -> np.ndarray:
    """Exact widening of an array of bf16 bit patterns, through the oracle's own scalar routine."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def f32_array_to_bf16(x) -> np.ndarray:
    """Round-to-nearest-even narrowing of an fp32 array (same rule as or_f32_to_bf16)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)
