"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol the
header declares, rejects bad arguments with the documented status codes before touching the
device, and its host helpers agree with the oracle."""
import ctypes as C
import os
import re

import numpy as np
import pytest
import torch

from conftest import ROOT
from weight_quantization_b200 import inputs

WQ_OK, WQ_ERR_NULL, WQ_ERR_SHAPE, WQ_ERR_DTYPE, WQ_ERR_ALIGN, WQ_ERR_BITS, WQ_ERR_NOT_QUANTIZABLE = 0, -1, -2, -3, -4, -5, -6


@pytest.fixture(scope="module")
def wq():
    from weight_quantization_b200 import build, ops
    build.build()
    return ops


def header_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(wq):
    names = header_functions()
    assert len(names) >= 11, names
    L = C.CDLL(wq.LIB_PATH)
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert set(names) <= set(wq.PROTOTYPES), set(names) - set(wq.PROTOTYPES)


def test_version_and_status_strings(wq):
    L = wq.lib()
    assert L.wq_version() >= 1
    for st in range(-7, 1):
        assert L.wq_status_string(st)
    assert L.wq_status_string(99) == b"unknown status"


def test_tq3_argument_validation(wq):
    L = wq.lib()
    m = np.zeros(4, np.uint32)
    mp = m.ctypes.data
    A = 0x10000  # a 16-byte aligned fake device address: validation fails before any use
    assert L.tq3_encode(A, 1, 0, mp, A, A, A, None) == WQ_OK          # empty: nothing enqueued
    assert L.tq3_encode(None, 1, 0, None, None, None, None, None) == WQ_OK
    assert L.tq3_encode(A, 1, -1, mp, A, A, A, None) == WQ_ERR_SHAPE
    assert L.tq3_encode(A, 7, 4, mp, A, A, A, None) == WQ_ERR_DTYPE
    assert L.tq3_encode(None, 1, 4, mp, A, A, A, None) == WQ_ERR_NULL
    assert L.tq3_encode(A, 1, 4, None, A, A, A, None) == WQ_ERR_NULL
    assert L.tq3_encode(A + 8, 1, 4, mp, A, A, A, None) == WQ_ERR_ALIGN
    assert L.tq3_encode(A, 1, 4, mp, A + 4, A, A, None) == WQ_ERR_ALIGN
    assert L.tq3_encode(A, 1, 4, mp, A, A + 2, A, None) == WQ_ERR_ALIGN
    assert L.tq3_decode(A, A, A, 0, mp, A, 0, None) == WQ_OK
    assert L.tq3_decode(A, A, A, -3, mp, A, 0, None) == WQ_ERR_SHAPE
    assert L.tq3_decode(A, A, A, 3, mp, A, 5, None) == WQ_ERR_DTYPE
    assert L.tq3_decode(A, None, A, 3, mp, A, 0, None) == WQ_ERR_NULL
    assert L.tq3_decode(A, A, A, 3, mp, A + 4, 0, None) == WQ_ERR_ALIGN
    assert L.tq3_compressed_bytes(10) == 560
    assert L.tq3_compressed_bytes(-1) == -1


def test_rpbh_argument_validation(wq):
    L = wq.lib()
    cb = np.zeros(16, np.float32).ctypes.data
    A = 0x10000
    q = lambda W=A, dt=1, rows=4, d=3072, perm=A, signs=A, bits=3, cbp=cb, packed=A, norms=A: \
        L.rpbh_quantize_weight(W, dt, rows, d, perm, signs, bits, cbp, packed, norms, None)
    assert q(rows=0) == WQ_OK
    assert q(rows=-1) == WQ_ERR_SHAPE
    assert q(d=0) == WQ_ERR_SHAPE
    assert q(d=100) == WQ_ERR_NOT_QUANTIZABLE     # 100 & -100 = 4 < 32
    assert q(d=48) == WQ_ERR_NOT_QUANTIZABLE      # 16 < 32
    assert q(d=WQ_MAX_D * 2) == WQ_ERR_SHAPE
    assert q(bits=1) == WQ_ERR_BITS and q(bits=5) == WQ_ERR_BITS
    assert q(dt=3) == WQ_ERR_DTYPE
    assert q(W=None) == WQ_ERR_NULL and q(cbp=None) == WQ_ERR_NULL and q(norms=None) == WQ_ERR_NULL
    assert q(W=A + 8) == WQ_ERR_ALIGN and q(packed=A + 2) == WQ_ERR_ALIGN
    dq = lambda unrot=1, perm=A, signs=A, bits=3, nd=1, od=0, out=A, d=3072: \
        L.rpbh_dequantize_weight(A, A, nd, 4, d, bits, cb, perm, signs, unrot, out, od, None)
    assert dq(perm=None) == WQ_ERR_NULL
    assert dq(bits=6) == WQ_ERR_BITS
    assert dq(od=9) == WQ_ERR_DTYPE
    assert dq(out=A + 4) == WQ_ERR_ALIGN
    assert dq(d=96 + 8) == WQ_ERR_NOT_QUANTIZABLE
    r = lambda x=A, d=3072, dt=1: L.rpbh_rotate_activations(x, dt, 4, d, A, A, A, None)
    assert r(x=None) == WQ_ERR_NULL and r(d=40) == WQ_ERR_NOT_QUANTIZABLE and r(dt=2) == WQ_ERR_DTYPE
    assert L.rpbh_packed_bytes(4096, 11008, 3) == 4096 * 11008 * 3 // 8
    assert L.rpbh_packed_bytes(1, 5, 3) == 3 and L.rpbh_packed_bytes(-1, 5, 3) == -1


WQ_MAX_D = 32768


def test_lloyd_max_host_helper_matches_oracle(wq, oracle):
    for bits in (1, 2, 3, 4):
        assert np.array_equal(wq.gaussian_lloyd_max(bits), oracle.gaussian_lloyd_max(bits))
    for bits in (2, 3, 4):
        for d in (32, 96, 3072, 11008):
            assert np.array_equal(wq.rpbh_codebook(bits, d), oracle.rpbh_codebook(bits, d))
    from conftest import read_golden
    for parts in read_golden("lloyd_max_fp32.txt"):  # and against the independent fp32 bit patterns
        want = np.array([int(v, 16) for v in parts[1:]], dtype=np.uint32)
        assert np.array_equal(wq.gaussian_lloyd_max(int(parts[0])).view(np.uint32), want)
    with pytest.raises(wq.WQError):
        wq.gaussian_lloyd_max(5)
    with pytest.raises(wq.WQError):
        wq.rpbh_codebook(3, 0)


def test_sign_mask_layout(wq):
    bits = inputs.tq3_sign_bits()
    m = wq.sign_mask_words(bits)
    assert np.array_equal(m, inputs.tq3_sign_mask_words(bits))
    assert [hex(v) for v in m] == ["0x3fd74222", "0x1ab7c17", "0xff4abaf6", "0x656b5fe7"]


def test_record_pool_and_attention_argument_validation(wq):
    """tq3_encode_aos / tq3_decode_aos / tq3_encode_slots / tq3_decode_paged / tq3_attention reject bad
    arguments with their documented codes before any device work (fake device addresses)."""
    L = wq.lib()
    m = np.zeros(4, np.uint32)
    mp = m.ctypes.data
    A = 0x10000
    assert L.tq3_encode_aos(A, 1, 0, mp, A, None) == WQ_OK
    assert L.tq3_encode_aos(A, 1, -1, mp, A, None) == WQ_ERR_SHAPE
    assert L.tq3_encode_aos(A, 1, 4, mp, A + 4, None) == WQ_ERR_ALIGN      # records need 8 bytes
    assert L.tq3_decode_aos(A, 4, mp, A + 8, 1, None) == WQ_ERR_ALIGN      # out needs 16 bytes
    assert L.tq3_decode_aos(None, 4, mp, A, 1, None) == WQ_ERR_NULL

    slots = lambda x=A, dt=1, n=4, msk=mp, sl=A, pool=A, n_pool=8: L.tq3_encode_slots(x, dt, n, msk, sl, pool, n_pool, None)
    assert slots(n=0) == WQ_OK
    assert slots(n=-1) == WQ_ERR_SHAPE
    assert slots(n_pool=-1) == WQ_ERR_SHAPE
    assert slots(dt=9) == WQ_ERR_DTYPE
    assert slots(sl=None) == WQ_ERR_NULL
    assert slots(pool=A + 4) == WQ_ERR_ALIGN
    assert slots(sl=A + 4) == WQ_ERR_ALIGN
    assert slots(x=A + 8) == WQ_ERR_ALIGN

    paged = lambda pool=A, n_pool=64, tab=A, n_pages=4, ps=16, n=64, out=A, dt=1: \
        L.tq3_decode_paged(pool, n_pool, tab, n_pages, ps, n, mp, out, dt, None)
    assert paged(n=0) == WQ_OK
    for ps in (0, 12, 3, 1 << 31):
        assert paged(ps=ps) == WQ_ERR_SHAPE                                # a power of two, 1 .. 2^30
    assert paged(n=65) == WQ_ERR_SHAPE                                     # more than the table covers
    assert paged(n_pages=-1) == WQ_ERR_SHAPE
    assert paged(dt=2) == WQ_ERR_DTYPE
    assert paged(tab=None) == WQ_ERR_NULL
    assert paged(tab=A + 2) == WQ_ERR_ALIGN
    assert paged(pool=A + 4) == WQ_ERR_ALIGN
    assert paged(out=A + 8) == WQ_ERR_ALIGN

    attn = lambda q=A, qdt=1, heads=2, rows=4, k=A, v=A, S=100, scale=0.088, out=A, odt=1: \
        L.tq3_attention(q, qdt, heads, rows, k, v, S, mp, scale, out, odt, None)
    assert attn(heads=0) == WQ_OK
    for rows in (0, (1 << 20) + 1):                                       # 1 .. 2^20 rows (chunks of 16)
        assert attn(rows=rows) == WQ_ERR_SHAPE
    for S in (0, (1 << 31) + 1):
        assert attn(S=S) == WQ_ERR_SHAPE
    assert attn(heads=-1) == WQ_ERR_SHAPE
    assert attn(scale=float("inf")) == WQ_ERR_SHAPE
    assert attn(scale=float("nan")) == WQ_ERR_SHAPE
    assert attn(qdt=5) == WQ_ERR_DTYPE
    assert attn(v=None) == WQ_ERR_NULL
    assert attn(k=A + 4) == WQ_ERR_ALIGN
    assert attn(q=A + 1) == WQ_ERR_ALIGN                                   # bf16 needs 2 bytes
    assert attn(out=A + 2, odt=0) == WQ_ERR_ALIGN                          # fp32 needs 4 bytes

    pa = lambda q=A, heads=2, rows=4, k=A, v=A, n_pool=64, tab=A, pph=4, ps=16, S=60, scale=0.088, out=A: \
        L.tq3_attention_paged(q, 1, heads, rows, k, v, n_pool, tab, pph, ps, S, mp, scale, out, 1, None)
    assert pa(heads=0) == WQ_OK
    assert pa(S=65) == WQ_ERR_SHAPE                                        # more than the table covers
    for ps in (0, 12, 1 << 31):
        assert pa(ps=ps) == WQ_ERR_SHAPE
    assert pa(n_pool=-1) == WQ_ERR_SHAPE
    assert pa(pph=-1) == WQ_ERR_SHAPE
    assert pa(scale=float("nan")) == WQ_ERR_SHAPE
    assert pa(tab=None) == WQ_ERR_NULL
    assert pa(tab=A + 2) == WQ_ERR_ALIGN
    assert pa(k=A + 4) == WQ_ERR_ALIGN


def test_bindings_reject_buffers_smaller_than_the_call(wq):
    """The C ABI takes plain pointers, so the Python binding checks every caller-supplied buffer's
    size first: a short one raises ValueError before any device work (CPU tensors suffice)."""
    mask = np.zeros(4, np.uint32)
    p, n, s = torch.zeros(4, 48, dtype=torch.uint8), torch.zeros(4), torch.zeros(4)
    with pytest.raises(ValueError, match="out holds"):
        wq.tq3_decode(p, n, s, mask, out=torch.empty(4 * 128 - 1))
    with pytest.raises(ValueError, match="packed holds"):
        wq.tq3_encode(torch.zeros(4, 128), mask, packed=torch.empty(4 * 48 - 1, dtype=torch.uint8))
    with pytest.raises(ValueError, match="records holds"):
        wq.tq3_encode_aos(torch.zeros(4, 128), mask, records=torch.empty(4 * 56 - 8, dtype=torch.uint8))
    with pytest.raises(ValueError, match="out holds"):
        wq.tq3_decode_aos(torch.zeros(4, 56, dtype=torch.uint8), mask, out=torch.empty(3, 128))
    with pytest.raises(ValueError, match="out holds"):
        wq.tq3_decode_paged(torch.zeros(64, 56, dtype=torch.uint8), torch.zeros(4, dtype=torch.int32), 16, 64, mask,
                            out=torch.empty(63, 128))
    rec = torch.zeros(2, 10, 56, dtype=torch.uint8)
    with pytest.raises(ValueError, match="out holds"):
        wq.tq3_attention(torch.zeros(2, 4, 128), rec, rec, mask, out=torch.empty(2, 3, 128))
    perm, signs = torch.zeros(63, dtype=torch.int32), torch.ones(64, dtype=torch.int8)
    with pytest.raises(ValueError, match="perm holds"):
        wq.rpbh_rotate_activations(torch.zeros(4, 64), perm, signs)
    cb = np.linspace(-1, 1, 8, dtype=np.float32)
    with pytest.raises(ValueError, match="packed holds"):
        wq.rpbh_dequantize_weight(torch.zeros(95, dtype=torch.uint8), torch.zeros(4), 4, 64, 3, cb)
    with pytest.raises(ValueError, match="row_norms holds"):
        wq.rpbh_linear(torch.zeros(96, dtype=torch.uint8), torch.zeros(3), 4, 64, 3, cb, torch.zeros(2, 64))


def test_bindings_reject_buffers_on_another_device_or_dtype(wq):
    """A caller-supplied buffer is written through a raw pointer on the stream of the call's main
    operand, so the binding rejects one that lives on another device or has a dtype the call does
    not take ("meta" tensors stand in for a second device on a CPU-only host)."""
    mask = np.zeros(4, np.uint32)
    rec = torch.zeros(2, 10, 56, dtype=torch.uint8)
    q = torch.zeros(2, 4, 128)
    with pytest.raises(ValueError, match="out must be on"):
        wq.tq3_attention(q, rec, rec, mask, out=torch.empty(2, 4, 128, device="meta"))
    with pytest.raises(ValueError, match="out must be one of"):
        wq.tq3_attention(q, rec, rec, mask, out=torch.empty(2, 4, 128, dtype=torch.int32))
    with pytest.raises(ValueError, match="k_records must be on"):
        wq.tq3_attention(q, rec.to("meta"), rec, mask)
    pool, table = torch.zeros(64, 56, dtype=torch.uint8), torch.zeros(4, dtype=torch.int32)
    with pytest.raises(ValueError, match="out must be on"):
        wq.tq3_decode_paged(pool, table, 16, 64, mask, out=torch.empty(64, 128, device="meta"))
    with pytest.raises(ValueError, match="out must be one of"):
        wq.tq3_decode_paged(pool, table, 16, 64, mask, out=torch.empty(64, 128, dtype=torch.float16))
    with pytest.raises(ValueError, match="page_table must be on"):
        wq.tq3_decode_paged(pool, table.to("meta"), 16, 64, mask)
    p, n, s = torch.zeros(4, 48, dtype=torch.uint8), torch.zeros(4), torch.zeros(4)
    with pytest.raises(ValueError, match="out must be on"):
        wq.tq3_decode(p, n, s, mask, out=torch.empty(4, 128, device="meta"))
    with pytest.raises(ValueError, match="norms must be on"):
        wq.tq3_decode(p, n.to("meta"), s, mask)
    with pytest.raises(ValueError, match="packed must be on"):
        wq.tq3_encode(torch.zeros(4, 128), mask, packed=torch.empty(4, 48, dtype=torch.uint8, device="meta"))
    perm, signs = torch.zeros(64, dtype=torch.int32), torch.ones(64, dtype=torch.int8)
    with pytest.raises(ValueError, match="out must be one of"):
        wq.rpbh_rotate_activations(torch.zeros(4, 64), perm, signs, out=torch.empty(4, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="perm must be on"):
        wq.rpbh_rotate_activations(torch.zeros(4, 64), perm.to("meta"), signs)


def test_requantize_and_code_packing_argument_validation(wq):
    """rpbh_requantize_weight checks the norm dtype and its alignment; rpbh_pack_codes and
    rpbh_unpack_codes check sizes, bits and pointers, all before any device work."""
    L = wq.lib()
    WQ_ERR_BITS = -5
    A = 0x10000
    cb = np.linspace(-1, 1, 8, dtype=np.float32)
    rq = lambda w=A, wdt=0, rows=4, d=64, bits=3, norms=A, ndt=1: L.rpbh_requantize_weight(
        w, wdt, rows, d, A, A, bits, cb.ctypes.data, A, norms, ndt, None)
    assert rq(rows=0) == WQ_OK
    assert rq(ndt=7) == WQ_ERR_DTYPE
    assert rq(wdt=7) == WQ_ERR_DTYPE
    assert rq(norms=A + 1) == WQ_ERR_ALIGN                          # bf16 norms need 2 bytes
    assert rq(norms=A + 2, ndt=0) == WQ_ERR_ALIGN                   # fp32 norms need 4 bytes
    assert rq(norms=None) == WQ_ERR_NULL
    assert rq(d=40) == WQ_ERR_NOT_QUANTIZABLE
    assert rq(bits=5) == WQ_ERR_BITS
    for fn in (L.rpbh_pack_codes, L.rpbh_unpack_codes):
        assert fn(A, 0, 3, A, None) == WQ_OK
        assert fn(A, -1, 3, A, None) == WQ_ERR_SHAPE
        assert fn(A, 8, 0, A, None) == WQ_ERR_BITS
        assert fn(A, 8, 9, A, None) == WQ_ERR_BITS
        assert fn(None, 8, 3, A, None) == WQ_ERR_NULL
        assert fn(A, 8, 3, None, None) == WQ_ERR_NULL
