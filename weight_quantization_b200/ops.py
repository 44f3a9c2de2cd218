"""Thin Python binding of libwq_b200.so (argument marshalling only).

Every function here checks tensor placement, dtype and contiguity, allocates outputs with torch
when the caller does not pass them, and forwards raw pointers, sizes and the current CUDA stream
to the C ABI declared in include/wq.h. All compute happens in the library's CUDA kernels; there
is no CPU or PyTorch fallback, and a missing library raises at the first call.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwq_b200.so")

WQ_F32, WQ_BF16 = 0, 1
_DT = {torch.float32: WQ_F32, torch.bfloat16: WQ_BF16}

# C prototypes of include/wq.h: name -> (restype, argtypes)
_vp, _i64, _int = C.c_void_p, C.c_int64, C.c_int
PROTOTYPES = {
    "tq3_encode": (_int, [_vp, _int, _i64, _vp, _vp, _vp, _vp, _vp]),
    "tq3_encode_exact": (_int, [_vp, _int, _i64, _vp, _vp, _vp, _vp, _vp]),
    "tq3_decode": (_int, [_vp, _vp, _vp, _i64, _vp, _vp, _int, _vp]),
    "tq3_encode_aos": (_int, [_vp, _int, _i64, _vp, _vp, _vp]),
    "tq3_decode_aos": (_int, [_vp, _i64, _vp, _vp, _int, _vp]),
    "tq3_encode_slots": (_int, [_vp, _int, _i64, _vp, _vp, _vp, _i64, _vp]),
    "tq3_decode_paged": (_int, [_vp, _i64, _vp, _i64, _i64, _i64, _vp, _vp, _int, _vp]),
    "tq3_attention": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _i64, _vp, C.c_float, _vp, _int, _vp]),
    "tq3_attention_paged": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _i64, _vp, _i64, _i64, _i64, _vp, C.c_float,
                                   _vp, _int, _vp]),
    "tq3_compressed_bytes": (_i64, [_i64]),
    "rpbh_quantize_weight": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _int, _vp, _vp, _vp, _vp]),
    "rpbh_requantize_weight": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _int, _vp, _vp, _vp, _int, _vp]),
    "rpbh_pack_codes": (_int, [_vp, _i64, _int, _vp, _vp]),
    "rpbh_unpack_codes": (_int, [_vp, _i64, _int, _vp, _vp]),
    "rpbh_dequantize_weight": (_int, [_vp, _vp, _int, _i64, _i64, _int, _vp, _vp, _vp, _int, _vp, _int, _vp]),
    "rpbh_rotate_activations": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _vp, _vp]),
    "rpbh_linear": (_int, [_vp, _vp, _int, _i64, _i64, _int, _vp, _vp, _i64, _vp, _vp, _vp]),
    "rpbh_packed_bytes": (_i64, [_i64, _i64, _int]),
    "wq_gaussian_lloyd_max": (_int, [_int, _int, _vp]),
    "wq_rpbh_codebook": (_int, [_int, _i64, _vp]),
    "wq_device_fault": (_int, [_vp]),
    "wq_selftest_wait_timeout": (_int, [_vp]),
    "wq_status_string": (C.c_char_p, [_int]),
    "wq_version": (_int, []),
}

_lib = None


class WQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {lib().wq_status_string(status).decode()} (status {status})")
        self.status = status


def lib():
    """Load the CUDA library (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libwq_b200.so not found at {LIB_PATH}: build it with "
                               "`python -m weight_quantization_b200.build` (there is no fallback)")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in PROTOTYPES.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def _check(fn: str, status: int):
    if status != 0:
        raise WQError(fn, status)


def _dev(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _fits(t, n: int, name: str):
    """The library takes plain pointers: a buffer smaller than what the call reads or writes is
    rejected here, before any device work."""
    if t is not None and t.numel() < n:
        raise ValueError(f"{name} holds {t.numel()} elements; the call needs {n}")


def _on(t, device, name: str, dtypes=None):
    """A caller-supplied buffer must live on the device whose stream the call is enqueued on (the
    library writes it through a raw pointer from that context) and have a dtype the call takes."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or t.device != torch.device(device):
        raise ValueError(f"{name} must be on {device}")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name} must be one of {sorted(str(d) for d in dtypes)}")


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def sign_mask_words(sign_bits) -> np.ndarray:
    """Lay out 128 sign draws (1 = +1, 0 = -1) as the four host words the ABI takes."""
    bits = np.asarray(sign_bits, dtype=np.uint64).reshape(4, 32)
    return (bits << np.arange(32, dtype=np.uint64)).sum(axis=1).astype(np.uint32)


def _mask_arg(mask) -> np.ndarray:
    m = np.ascontiguousarray(np.asarray(mask, dtype=np.uint32))
    if m.shape != (4,):
        raise ValueError("sign mask must be 4 uint32 words")
    return m


# ---------------------------------------------------------------------------------------------
# TQ3
# ---------------------------------------------------------------------------------------------
def tq3_encode(x: torch.Tensor, sign_mask, packed=None, norms=None, scales=None, exact=False):
    """TQ3-encode a [..., D] fp32/bf16 CUDA tensor (D a multiple of 128).

    Returns (packed uint8 [..., D/128, 48], norms fp32 [..., D/128], scales fp32 [..., D/128]).
    exact=True calls tq3_encode_exact (the page's rounding bit for bit) instead of tq3_encode.
    """
    if x.dtype not in _DT:
        raise ValueError("x must be float32 or bfloat16")
    if x.ndim == 0 or x.shape[-1] % 128 != 0 or x.shape[-1] <= 0:
        raise ValueError("last dim must be a positive multiple of 128")
    lead = tuple(x.shape[:-1]) + (x.shape[-1] // 128,)
    n_vec = x.numel() // 128
    if packed is None:
        packed = torch.empty(lead + (48,), dtype=torch.uint8, device=x.device)
    if norms is None:
        norms = torch.empty(lead, dtype=torch.float32, device=x.device)
    if scales is None:
        scales = torch.empty(lead, dtype=torch.float32, device=x.device)
    for name, t in (("packed", packed), ("norms", norms), ("scales", scales)):
        _on(t, x.device, name)
    _fits(packed, 48 * n_vec, "packed")
    _fits(norms, n_vec, "norms")
    _fits(scales, n_vec, "scales")
    m = _mask_arg(sign_mask)
    name = "tq3_encode_exact" if exact else "tq3_encode"
    st = getattr(lib(), name)(_dev(x, "x"), _DT[x.dtype], n_vec, m.ctypes.data, _dev(packed, "packed"),
                              _dev(norms, "norms"), _dev(scales, "scales"), _stream(x.device))
    _check(name, st)
    return packed, norms, scales


def tq3_decode(packed: torch.Tensor, norms: torch.Tensor, scales: torch.Tensor, sign_mask,
               out_dtype=torch.float32, out=None):
    """Decode TQ3 records back to [..., 128] values of out_dtype (fp32 or bf16)."""
    if packed.shape[-1] != 48 or tuple(packed.shape[:-1]) != tuple(norms.shape) or norms.shape != scales.shape:
        raise ValueError("packed must be [..., 48] with norms/scales of shape [...]")
    n_vec = norms.numel()
    if out is None:
        out = torch.empty(tuple(norms.shape) + (128,), dtype=out_dtype, device=packed.device)
    for name, t in (("norms", norms), ("scales", scales)):
        _on(t, packed.device, name)
    _on(out, packed.device, "out", _DT)
    _fits(out, 128 * n_vec, "out")
    m = _mask_arg(sign_mask)
    st = lib().tq3_decode(_dev(packed, "packed"), _dev(norms, "norms"), _dev(scales, "scales"), n_vec,
                          m.ctypes.data, _dev(out, "out"), _DT[out.dtype], _stream(packed.device))
    _check("tq3_decode", st)
    return out


def tq3_encode_aos(x: torch.Tensor, sign_mask, records=None):
    """TQ3-encode a [..., D] fp32/bf16 CUDA tensor into 56-byte records [..., D/128, 56] (the packed
    bytes, the fp32 norm, the fp32 scale)."""
    if x.dtype not in _DT:
        raise ValueError("x must be float32 or bfloat16")
    if x.ndim == 0 or x.shape[-1] % 128 != 0 or x.shape[-1] <= 0:
        raise ValueError("last dim must be a positive multiple of 128")
    lead = tuple(x.shape[:-1]) + (x.shape[-1] // 128,)
    if records is None:
        records = torch.empty(lead + (56,), dtype=torch.uint8, device=x.device)
    _on(records, x.device, "records")
    _fits(records, 56 * (x.numel() // 128), "records")
    m = _mask_arg(sign_mask)
    st = lib().tq3_encode_aos(_dev(x, "x"), _DT[x.dtype], x.numel() // 128, m.ctypes.data, _dev(records, "records"),
                              _stream(x.device))
    _check("tq3_encode_aos", st)
    return records


def tq3_decode_aos(records: torch.Tensor, sign_mask, out_dtype=torch.float32, out=None):
    """Decode 56-byte TQ3 records [..., 56] back to [..., 128] values of out_dtype (fp32 or bf16)."""
    if records.shape[-1] != 56:
        raise ValueError("records must be [..., 56]")
    n_vec = records.numel() // 56
    if out is None:
        out = torch.empty(tuple(records.shape[:-1]) + (128,), dtype=out_dtype, device=records.device)
    _on(out, records.device, "out", _DT)
    _fits(out, 128 * n_vec, "out")
    m = _mask_arg(sign_mask)
    st = lib().tq3_decode_aos(_dev(records, "records"), n_vec, m.ctypes.data, _dev(out, "out"), _DT[out.dtype],
                              _stream(records.device))
    _check("tq3_decode_aos", st)
    return out


def tq3_encode_slots(x: torch.Tensor, sign_mask, slots: torch.Tensor, pool: torch.Tensor):
    """TQ3-encode the vectors of x ([..., D] fp32/bf16, D a multiple of 128, so x.numel() / 128
    vectors) into a pool of 56-byte records [n_pool, 56]: vector v goes to record slots[v] (int64;
    a negative slot skips the vector). Slots at or beyond n_pool are skipped and raise device fault
    bit 6. Returns pool."""
    if x.dtype not in _DT:
        raise ValueError("x must be float32 or bfloat16")
    if x.ndim == 0 or x.shape[-1] % 128 != 0 or x.shape[-1] <= 0:
        raise ValueError("last dim must be a positive multiple of 128")
    n_vec = x.numel() // 128
    if slots.dtype != torch.int64 or slots.numel() != n_vec:
        raise ValueError("slots must be int64 with one entry per vector")
    if pool.dtype != torch.uint8 or pool.ndim != 2 or pool.shape[1] != 56:
        raise ValueError("pool must be uint8 [n_pool, 56]")
    _on(slots, x.device, "slots")
    _on(pool, x.device, "pool")
    m = _mask_arg(sign_mask)
    st = lib().tq3_encode_slots(_dev(x, "x"), _DT[x.dtype], n_vec, m.ctypes.data, _dev(slots, "slots"),
                                _dev(pool, "pool"), pool.shape[0], _stream(x.device))
    _check("tq3_encode_slots", st)
    return pool


def tq3_decode_paged(pool: torch.Tensor, page_table: torch.Tensor, page_size: int, n_vec: int, sign_mask,
                     out_dtype=torch.float32, out=None):
    """Decode n_vec logically consecutive vectors from a pool of 56-byte records [n_pool, 56]
    through a page table (int32): vector p is record page_table[p // page_size] * page_size +
    p % page_size. page_size is a power of two. Returns [n_vec, 128] of out_dtype; entries outside
    the pool decode as zeros and raise device fault bit 6."""
    if pool.dtype != torch.uint8 or pool.ndim != 2 or pool.shape[1] != 56:
        raise ValueError("pool must be uint8 [n_pool, 56]")
    if page_table.dtype != torch.int32:
        raise ValueError("page_table must be int32")
    if out is None:
        out = torch.empty((n_vec, 128), dtype=out_dtype, device=pool.device)
    _on(page_table, pool.device, "page_table")
    _on(out, pool.device, "out", _DT)
    _fits(out, 128 * n_vec, "out")
    m = _mask_arg(sign_mask)
    st = lib().tq3_decode_paged(_dev(pool, "pool"), pool.shape[0], _dev(page_table, "page_table"),
                                page_table.numel(), int(page_size), int(n_vec), m.ctypes.data, _dev(out, "out"),
                                _DT[out.dtype], _stream(pool.device))
    _check("tq3_decode_paged", st)
    return out


def tq3_attention(q: torch.Tensor, k_records: torch.Tensor, v_records: torch.Tensor, sign_mask,
                  softmax_scale: float = 128 ** -0.5, out_dtype=None, out=None):
    """Attention of q [heads, m, 128] (fp32/bf16; the m rows of a head share its keys and values,
    e.g. the query heads of one KV head) over TQ3 records k_records, v_records [heads, S, 56]:
    softmax(softmax_scale * q k^T) v with k, v the decoded records. Returns [heads, m, 128]."""
    if q.dtype not in _DT or q.ndim != 3 or q.shape[2] != 128:
        raise ValueError("q must be [heads, m, 128] float32 or bfloat16")
    heads, m = q.shape[0], q.shape[1]
    for name, t in (("k_records", k_records), ("v_records", v_records)):
        if t.dtype != torch.uint8 or t.ndim != 3 or t.shape[0] != heads or t.shape[2] != 56:
            raise ValueError(f"{name} must be uint8 [heads, S, 56]")
    if k_records.shape != v_records.shape:
        raise ValueError("k_records and v_records must have the same shape")
    if out is None:
        out = torch.empty((heads, m, 128), dtype=out_dtype or q.dtype, device=q.device)
    _on(k_records, q.device, "k_records")
    _on(v_records, q.device, "v_records")
    _on(out, q.device, "out", _DT)
    _fits(out, heads * m * 128, "out")
    msk = _mask_arg(sign_mask)
    st = lib().tq3_attention(_dev(q, "q"), _DT[q.dtype], heads, m, _dev(k_records, "k_records"),
                             _dev(v_records, "v_records"), k_records.shape[1], msk.ctypes.data,
                             float(softmax_scale), _dev(out, "out"), _DT[out.dtype], _stream(q.device))
    _check("tq3_attention", st)
    return out


def tq3_attention_paged(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor, page_table: torch.Tensor,
                        page_size: int, S: int, sign_mask, softmax_scale: float = 128 ** -0.5, out_dtype=None,
                        out=None):
    """tq3_attention over a paged cache: q [heads, m, 128]; k_pool, v_pool [n_pool, 56] records;
    page_table int32 [heads, pages_per_head]; key j of head h is record
    page_table[h, j // page_size] * page_size + j % page_size. Returns [heads, m, 128]."""
    if q.dtype not in _DT or q.ndim != 3 or q.shape[2] != 128:
        raise ValueError("q must be [heads, m, 128] float32 or bfloat16")
    heads, m = q.shape[0], q.shape[1]
    for name, t in (("k_pool", k_pool), ("v_pool", v_pool)):
        if t.dtype != torch.uint8 or t.ndim != 2 or t.shape[1] != 56:
            raise ValueError(f"{name} must be uint8 [n_pool, 56]")
    if k_pool.shape != v_pool.shape:
        raise ValueError("k_pool and v_pool must have the same shape")
    if page_table.dtype != torch.int32 or page_table.ndim != 2 or page_table.shape[0] != heads:
        raise ValueError("page_table must be int32 [heads, pages_per_head]")
    if out is None:
        out = torch.empty((heads, m, 128), dtype=out_dtype or q.dtype, device=q.device)
    for name, t in (("k_pool", k_pool), ("v_pool", v_pool), ("page_table", page_table)):
        _on(t, q.device, name)
    _on(out, q.device, "out", _DT)
    _fits(out, heads * m * 128, "out")
    msk = _mask_arg(sign_mask)
    st = lib().tq3_attention_paged(_dev(q, "q"), _DT[q.dtype], heads, m, _dev(k_pool, "k_pool"),
                                   _dev(v_pool, "v_pool"), k_pool.shape[0], _dev(page_table, "page_table"),
                                   page_table.shape[1], int(page_size), int(S), msk.ctypes.data, float(softmax_scale),
                                   _dev(out, "out"), _DT[out.dtype], _stream(q.device))
    _check("tq3_attention_paged", st)
    return out


def tq3_compressed_bytes(n_vec: int) -> int:
    return int(lib().tq3_compressed_bytes(n_vec))


# ---------------------------------------------------------------------------------------------
# RPBH
# ---------------------------------------------------------------------------------------------
def _codebook_arg(codebook, bits) -> np.ndarray:
    cb = np.ascontiguousarray(np.asarray(codebook, dtype=np.float32))
    if cb.shape != (1 << bits,):
        raise ValueError(f"codebook must hold {1 << bits} floats")
    return cb


def rpbh_packed_bytes(rows: int, d: int, bits: int) -> int:
    return int(lib().rpbh_packed_bytes(rows, d, bits))


def rpbh_quantize_weight(W: torch.Tensor, perm: torch.Tensor, signs: torch.Tensor, bits: int, codebook,
                         packed=None, row_norms=None):
    """Quantize W [rows, d] (fp32/bf16). Returns (packed uint8 bitstream, row_norms in W's dtype)."""
    rows, d = W.shape
    cb = _codebook_arg(codebook, bits)
    if packed is None:
        packed = torch.empty(max(rpbh_packed_bytes(rows, d, bits), 0), dtype=torch.uint8, device=W.device)
    if row_norms is None:
        row_norms = torch.empty(rows, dtype=W.dtype, device=W.device)
    for name, t in (("packed", packed), ("row_norms", row_norms), ("perm", perm), ("signs", signs)):
        _on(t, W.device, name)
    _fits(packed, rpbh_packed_bytes(rows, d, bits), "packed")
    _fits(row_norms, rows, "row_norms")
    _fits(perm, d, "perm")
    _fits(signs, d, "signs")
    st = lib().rpbh_quantize_weight(_dev(W, "W"), _DT.get(W.dtype, -1), rows, d, _dev(perm, "perm"),
                                    _dev(signs, "signs"), bits, cb.ctypes.data, _dev(packed, "packed"),
                                    _dev(row_norms, "row_norms"), _stream(W.device))
    _check("rpbh_quantize_weight", st)
    return packed, row_norms


def rpbh_requantize_weight(W: torch.Tensor, perm: torch.Tensor, signs: torch.Tensor, bits: int, codebook,
                           norm_dtype, packed=None, row_norms=None):
    """requantize_: quantize W [rows, d] (fp32/bf16) with the stored perm, signs and codebook, the
    row norms in norm_dtype (the module's original dtype). Returns (packed, row_norms)."""
    rows, d = W.shape
    cb = _codebook_arg(codebook, bits)
    if norm_dtype not in _DT:
        raise ValueError("norm_dtype must be torch.float32 or torch.bfloat16")
    if packed is None:
        packed = torch.empty(max(rpbh_packed_bytes(rows, d, bits), 0), dtype=torch.uint8, device=W.device)
    if row_norms is None:
        row_norms = torch.empty(rows, dtype=norm_dtype, device=W.device)
    for name, t in (("packed", packed), ("perm", perm), ("signs", signs)):
        _on(t, W.device, name)
    _on(row_norms, W.device, "row_norms", (norm_dtype,))
    _fits(packed, rpbh_packed_bytes(rows, d, bits), "packed")
    _fits(row_norms, rows, "row_norms")
    _fits(perm, d, "perm")
    _fits(signs, d, "signs")
    st = lib().rpbh_requantize_weight(_dev(W, "W"), _DT.get(W.dtype, -1), rows, d, _dev(perm, "perm"),
                                      _dev(signs, "signs"), bits, cb.ctypes.data, _dev(packed, "packed"),
                                      _dev(row_norms, "row_norms"), _DT[norm_dtype], _stream(W.device))
    _check("rpbh_requantize_weight", st)
    return packed, row_norms


def rpbh_pack_codes(codes: torch.Tensor, bits: int, packed=None):
    """pack_codes: codes (uint8, any shape, flattened) -> flat MSB-first stream of
    ceil(numel / 8) * bits bytes."""
    if codes.dtype != torch.uint8:
        raise ValueError("codes must be uint8")
    numel = codes.numel()
    nbytes = (numel + 7) // 8 * bits
    if packed is None:
        packed = torch.empty(nbytes, dtype=torch.uint8, device=codes.device)
    _on(packed, codes.device, "packed", (torch.uint8,))
    _fits(packed, nbytes, "packed")
    st = lib().rpbh_pack_codes(_dev(codes, "codes"), numel, bits, _dev(packed, "packed"), _stream(codes.device))
    _check("rpbh_pack_codes", st)
    return packed


def rpbh_unpack_codes(packed: torch.Tensor, bits: int, numel: int, codes=None):
    """unpack_codes: the first numel codes of a packed stream, as uint8 [numel]."""
    if packed.dtype != torch.uint8:
        raise ValueError("packed must be uint8")
    _fits(packed, (numel + 7) // 8 * bits, "packed")
    if codes is None:
        codes = torch.empty(numel, dtype=torch.uint8, device=packed.device)
    _on(codes, packed.device, "codes", (torch.uint8,))
    _fits(codes, numel, "codes")
    st = lib().rpbh_unpack_codes(_dev(packed, "packed"), numel, bits, _dev(codes, "codes"), _stream(packed.device))
    _check("rpbh_unpack_codes", st)
    return codes


def rpbh_dequantize_weight(packed: torch.Tensor, row_norms: torch.Tensor, rows: int, d: int, bits: int, codebook,
                           perm=None, signs=None, unrotate: bool = False, out_dtype=torch.float32, out=None):
    """Dequantize to [rows, d]: the rotated weight W P^T, or (unrotate=True) W itself."""
    cb = _codebook_arg(codebook, bits)
    if out is None:
        out = torch.empty(rows, d, dtype=out_dtype, device=packed.device)
    for name, t in (("row_norms", row_norms), ("perm", perm), ("signs", signs)):
        _on(t, packed.device, name)
    _on(out, packed.device, "out", _DT)
    _fits(packed, rpbh_packed_bytes(rows, d, bits), "packed")
    _fits(row_norms, rows, "row_norms")
    _fits(out, rows * d, "out")
    _fits(perm, d, "perm")
    _fits(signs, d, "signs")
    pp = _dev(perm, "perm") if perm is not None else None
    sp = _dev(signs, "signs") if signs is not None else None
    st = lib().rpbh_dequantize_weight(_dev(packed, "packed"), _dev(row_norms, "row_norms"),
                                      _DT.get(row_norms.dtype, -1), rows, d, bits, cb.ctypes.data, pp, sp,
                                      int(bool(unrotate)), _dev(out, "out"), _DT.get(out.dtype, -1),
                                      _stream(packed.device))
    _check("rpbh_dequantize_weight", st)
    return out


def rpbh_rotate_activations(x: torch.Tensor, perm: torch.Tensor, signs: torch.Tensor, out=None):
    """x_rot = blkdiag(H_h) D P x for every row of x [rows, d] (fp32/bf16)."""
    rows, d = x.shape
    if out is None:
        out = torch.empty_like(x)
    for name, t in (("perm", perm), ("signs", signs)):
        _on(t, x.device, name)
    _on(out, x.device, "out", (x.dtype,))
    _fits(out, rows * d, "out")
    _fits(perm, d, "perm")
    _fits(signs, d, "signs")
    st = lib().rpbh_rotate_activations(_dev(x, "x"), _DT.get(x.dtype, -1), rows, d, _dev(perm, "perm"),
                                       _dev(signs, "signs"), _dev(out, "out"), _stream(x.device))
    _check("rpbh_rotate_activations", st)
    return out


def rpbh_linear(packed: torch.Tensor, row_norms: torch.Tensor, out_features: int, d: int, bits: int, codebook,
                x_rot: torch.Tensor, bias=None, out=None):
    """y = x_rot W'^T + bias [m, out_features] bf16, W' the rotated dequantized weight of `packed`."""
    cb = _codebook_arg(codebook, bits)
    m = x_rot.shape[0]
    if out is None:
        out = torch.empty(m, out_features, dtype=torch.bfloat16, device=x_rot.device)
    for name, t in (("packed", packed), ("row_norms", row_norms), ("bias", bias)):
        _on(t, x_rot.device, name)
    _on(out, x_rot.device, "y", (torch.bfloat16,))
    _fits(packed, rpbh_packed_bytes(out_features, d, bits), "packed")
    _fits(row_norms, out_features, "row_norms")
    _fits(x_rot, m * d, "x_rot")
    _fits(bias, out_features, "bias")
    _fits(out, m * out_features, "y")
    bp = _dev(bias, "bias") if bias is not None else None
    st = lib().rpbh_linear(_dev(packed, "packed"), _dev(row_norms, "row_norms"), _DT.get(row_norms.dtype, -1),
                           out_features, d, bits, cb.ctypes.data, _dev(x_rot, "x_rot"), m, bp, _dev(out, "y"),
                           _stream(x_rot.device))
    _check("rpbh_linear", st)
    return out


# ---------------------------------------------------------------------------------------------
# host helpers
# ---------------------------------------------------------------------------------------------
def gaussian_lloyd_max(bits: int, iters: int = 200) -> np.ndarray:
    out = np.zeros(1 << bits, np.float32)
    _check("wq_gaussian_lloyd_max", lib().wq_gaussian_lloyd_max(bits, iters, out.ctypes.data))
    return out


def selftest_wait_timeout(device=None):
    """Runs the library's bounded-wait self-test on the current stream (about 2 s of GPU time)."""
    _check("wq_selftest_wait_timeout", lib().wq_selftest_wait_timeout(_stream(device or torch.cuda.current_device())))


def device_fault() -> int:
    """Read and clear the sticky fault bits (non-zero if a kernel's bounded TMA wait ran out)."""
    v = C.c_uint(0)
    _check("wq_device_fault", lib().wq_device_fault(C.byref(v)))
    return int(v.value)


def rpbh_codebook(bits: int, d: int) -> np.ndarray:
    out = np.zeros(1 << bits, np.float32)
    _check("wq_rpbh_codebook", lib().wq_rpbh_codebook(bits, d, out.ctypes.data))
    return out
