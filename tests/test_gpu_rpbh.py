"""GPU parity of the RPBH kernels against the oracle, through the C ABI (page "orbit_quant.py")."""
import numpy as np
import pytest
import torch

import parity
from weight_quantization_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wq():
    from weight_quantization_b200 import build, ops
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return ops


def _t(a, bf16=False):
    if bf16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _np16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _params(d):
    perm, signs = inputs.rpbh_params(d)
    return perm, signs, _t(perm), _t(signs)


def _quantize_and_check(wq, oracle, w, is_bf16, d, bits):
    perm, signs, perm_d, signs_d = _params(d)
    h = d & -d
    cb = oracle.rpbh_codebook(bits, d)
    packed, norms = wq.rpbh_quantize_weight(_t(w, is_bf16), perm_d, signs_d, bits, cb)
    st, _, ref_norms = parity.check_rpbh_quantize(oracle, w, is_bf16, perm, signs, h, cb, bits,
                                                  packed.cpu().numpy())
    if is_bf16:
        # stored in the weight dtype: one bf16 rounding of fp32 norms that agree to 1e-5
        ref16 = oracle.f32_array_to_bf16(ref_norms).astype(np.int64)
        got16 = _np16(norms).astype(np.int64)
        assert np.all(np.abs(got16 - ref16) <= 1)
        st["norms_equal"] = int((got16 == ref16).sum())
    else:
        st["norms_equal"] = parity.check_norms(norms.cpu().numpy(), ref_norms)
    return st, packed, norms


@pytest.mark.parametrize("d,rows", [(32, 5), (96, 37), (192, 11), (256, 3), (1024, 9), (3072, 17), (640, 1),
                                    (4096, 3), (12288, 2), (6400, 7), (9472, 5), (1536, 3), (6144, 2), (768, 4),
                                    (13056, 1), (13056, 3), (15360, 2)])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("is_bf16", [False, True])
def test_quantize_small(wq, oracle, d, rows, bits, is_bf16):
    w = inputs.gaussian((rows, d), seed=d * 7 + rows) * 0.02
    if rows > 2:
        w[1] = 0.0
    if is_bf16:
        w = inputs.to_bf16_bits(torch.from_numpy(w))
    st, _, _ = _quantize_and_check(wq, oracle, w, is_bf16, d, bits)
    assert st["code_mismatches"] == 0 and st["bytes_equal"] and st["norms_equal"] == rows, st


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quantize_llm_weight_full_size(wq, oracle, bits):
    """W[4096, 11008] bf16 (h = 256), every row checked."""
    w = _llm_weight()
    st, _, _ = _quantize_and_check(wq, oracle, w, True, 11008, bits)
    print("rpbh quantize C4", bits, st)
    # the same fp32 steps as the oracle, with fp64 norms: every code and every bf16 norm matches
    assert st["code_mismatches"] == 0 and st["bytes_equal"] and st["norms_equal"] == w.shape[0], st


_W4 = None


def _llm_weight():
    global _W4
    if _W4 is None:
        _W4 = inputs.llm_weight()
    return _W4


@pytest.mark.parametrize("rows", [3072, 12288])
def test_quantize_dit_weights_full_size(wq, oracle, rows):
    """DiT W[3072, 3072] and W[12288, 3072] bf16 (h = 1024) at 3 bits, every row checked."""
    w = inputs.dit_weight(rows)
    st, _, _ = _quantize_and_check(wq, oracle, w, True, 3072, 3)
    print("rpbh quantize C5", rows, st)
    assert st["code_mismatches"] == 0 and st["bytes_equal"] and st["norms_equal"] == rows, st


@pytest.mark.parametrize("d,rows,bits", [(96, 7, 2), (192, 3, 3), (1024, 5, 3), (3072, 33, 4), (11008, 4, 3),
                                         (4096, 2, 2), (1536, 3, 3), (6144, 2, 4)])
@pytest.mark.parametrize("norm_bf16", [False, True])
@pytest.mark.parametrize("out_bf16", [False, True])
@pytest.mark.parametrize("unrotate", [False, True])
def test_dequantize(wq, oracle, d, rows, bits, norm_bf16, out_bf16, unrotate):
    perm, signs, perm_d, signs_d = _params(d)
    h = d & -d
    cb = oracle.rpbh_codebook(bits, d)
    codes = inputs.uniform_int((rows, d), 1 << bits, seed=d + rows + bits)
    packed = oracle.pack_codes(codes, bits)
    norms32 = (np.abs(inputs.gaussian((rows,), seed=rows)) * 0.7 + 0.05).astype(np.float32)
    if norm_bf16:
        n16 = oracle.f32_array_to_bf16(norms32)
        norms_dev = _t(n16, True)
        norms_f32 = oracle.bf16_array_to_f32(n16)
    else:
        norms_dev = _t(norms32)
        norms_f32 = norms32
    out = wq.rpbh_dequantize_weight(_t(packed), norms_dev, rows, d, bits, cb, perm_d, signs_d, unrotate,
                                    out_dtype=torch.bfloat16 if out_bf16 else torch.float32)
    if unrotate:
        ref = oracle.rpbh_dequantize(packed, norms_f32, rows, d, bits, cb, np.argsort(perm).astype(np.int32), signs, h)
        if out_bf16:
            ref = oracle.f32_array_to_bf16(ref)
    else:
        ref = oracle.rpbh_dequantize_rotated(packed, norms_f32, rows, d, bits, cb, out_bf16=out_bf16)
    got = _np16(out) if out_bf16 else out.cpu().numpy()
    if out_bf16:
        r = parity.rel_rows(oracle.bf16_array_to_f32(got), oracle.bf16_array_to_f32(ref))
        assert r.max() <= parity.BF16_RTOL
    else:
        r = parity.rel_rows(got, ref)
        assert r.max() <= parity.F32_RTOL
    assert np.array_equal(got, ref), "expected bit-exact output (same fp32 steps as the oracle)"


def test_quantize_then_dequantize_llm_roundtrip(wq, oracle):
    """W'[r] P reconstructs W: row cosine at 3 bits near the Lloyd-Max value (~0.97)."""
    w = _llm_weight()[:256]
    perm, signs, perm_d, signs_d = _params(11008)
    cb = oracle.rpbh_codebook(3, 11008)
    wd = _t(w, True)
    packed, norms = wq.rpbh_quantize_weight(wd, perm_d, signs_d, 3, cb)
    back = wq.rpbh_dequantize_weight(packed, norms, 256, 11008, 3, cb, perm_d, signs_d, True)
    cos = torch.nn.functional.cosine_similarity(back.double(), wd.double(), dim=1)
    assert cos.mean().item() > 0.96


@pytest.mark.parametrize("rows,d", [(2048, 11008), (4096, 3072), (3, 96), (1, 32), (5, 192), (3, 4096),
                                    (7, 640), (9, 2880), (5, 6400), (3, 1536), (2, 6144), (3, 256), (4, 768),
                                    (2, 1024), (5, 13056), (3, 15360), (301, 3072)])
def test_rotate_activations(wq, oracle, rows, d):
    perm, signs, perm_d, signs_d = _params(d)
    h = d & -d
    x = inputs.activations(rows, d, seed=3 if d == 11008 else 4)
    out = wq.rpbh_rotate_activations(_t(x, True), perm_d, signs_d)
    got = _np16(out)
    ref = oracle.rpbh_rotate_bf16(x, perm, signs, h)
    r = parity.rel_rows(oracle.bf16_array_to_f32(got), oracle.bf16_array_to_f32(ref))
    assert r.max() <= parity.BF16_RTOL
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("rows,d", [(6, 6400), (4, 2880)])
def test_rotate_fp32_many_blocks(wq, oracle, rows, d):
    """fp32 rotation of rows with many h-blocks (25 blocks of 256; 45 blocks of 64), bit for bit."""
    perm, signs, perm_d, signs_d = _params(d)
    x = torch.from_numpy(inputs.gaussian((rows, d), seed=d + rows)).cuda()
    xr = wq.rpbh_rotate_activations(x, perm_d, signs_d)
    assert np.array_equal(xr.cpu().numpy(), oracle.rpbh_forward(x.cpu().numpy(), perm, signs, d & -d))


def test_rotate_fp32_and_matmul_invariance(wq, oracle):
    """(W P^T)(P x) = W x with fp32 rotations of both operands."""
    d = 3072
    perm, signs, perm_d, signs_d = _params(d)
    W = torch.from_numpy(inputs.gaussian((64, d), seed=5)).cuda()
    x = torch.from_numpy(inputs.gaussian((16, d), seed=6)).cuda()
    Wr = wq.rpbh_rotate_activations(W, perm_d, signs_d)
    xr = wq.rpbh_rotate_activations(x, perm_d, signs_d)
    ref = oracle.rpbh_forward(x.cpu().numpy(), perm, signs, d & -d)
    assert np.array_equal(xr.cpu().numpy(), ref)
    y = (Wr.double() @ xr.double().T)
    y0 = (W.double() @ x.double().T)
    assert torch.allclose(y, y0, atol=1e-3)


def test_rpbh_errors(wq):
    perm_d = torch.zeros(100, dtype=torch.int32, device="cuda")
    signs_d = torch.ones(100, dtype=torch.int8, device="cuda")
    with pytest.raises(wq.WQError) as e:
        wq.rpbh_rotate_activations(torch.zeros(4, 100, device="cuda"), perm_d, signs_d)
    assert e.value.status == -6


def test_asymmetric_codebook_takes_generic_bucketize(wq, oracle):
    """A caller-supplied codebook that is not antisymmetric is bucketized edge by edge."""
    d, rows, bits = 3072, 6, 3
    perm, signs, perm_d, signs_d = _params(d)
    cb = (oracle.rpbh_codebook(bits, d) + np.float32(0.001)).astype(np.float32)
    w = inputs.gaussian((rows, d), seed=91) * 0.02
    packed, norms = wq.rpbh_quantize_weight(_t(w), perm_d, signs_d, bits, cb)
    st, _, ref_norms = parity.check_rpbh_quantize(oracle, w, False, perm, signs, d & -d, cb, bits, packed.cpu().numpy())
    assert st["bytes_equal"]
    parity.check_norms(norms.cpu().numpy(), ref_norms)


def test_misaligned_tables_take_generic_path(wq, oracle):
    """perm/signs that are only 4-byte aligned still work (the general kernels take them)."""
    d, rows = 1024, 4
    perm, signs = inputs.rpbh_params(d)
    pbuf = torch.zeros(d + 1, dtype=torch.int32, device="cuda")
    pbuf[1:] = torch.from_numpy(perm).cuda()
    sbuf = torch.zeros(d + 1, dtype=torch.int8, device="cuda")
    sbuf[1:] = torch.from_numpy(signs).cuda()
    x = inputs.activations(rows, d, seed=92)
    out = wq.rpbh_rotate_activations(_t(x, True), pbuf[1:], sbuf[1:])
    assert np.array_equal(_np16(out), oracle.rpbh_rotate_bf16(x, perm, signs, d & -d))


# ------------------------------------------------------------------------------------------------
# requantize_ (norms in the module's original dtype) and pack_codes / unpack_codes on any length
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("d,rows", [(96, 37), (3072, 17), (11008, 5), (12288, 2), (6144, 3)])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("w_bf16,norm_bf16", [(False, True), (True, False), (False, False), (True, True)])
def test_requantize_norm_dtype(wq, oracle, d, rows, bits, w_bf16, norm_bf16):
    """Page "orbit_quant.py", requantize_: the new weight in fp32 (or bf16, which casts to fp32
    exactly) quantized with the stored tables, the norms in the module's original dtype."""
    w = inputs.gaussian((rows, d), seed=d + rows + bits) * 0.03
    w[0] *= 50.0
    if w_bf16:
        w = inputs.to_bf16_bits(torch.from_numpy(w))
    perm, signs, perm_d, signs_d = _params(d)
    cb = oracle.rpbh_codebook(bits, d)
    ndt = torch.bfloat16 if norm_bf16 else torch.float32
    packed, norms = wq.rpbh_requantize_weight(_t(w, w_bf16), perm_d, signs_d, bits, cb, ndt)
    torch.cuda.synchronize()
    assert norms.dtype == ndt and norms.shape == (rows,)
    st, ref_packed, ref_norms = parity.check_rpbh_quantize(oracle, w, w_bf16, perm, signs, d & -d, cb, bits,
                                                            packed.cpu().numpy())
    assert st["code_mismatches"] == 0 and st["bytes_equal"], st
    if norm_bf16:
        # one nearest-even rounding of the fp32 norm, which equals the oracle's
        ref16 = oracle.f32_array_to_bf16(ref_norms).astype(np.int64)
        assert np.array_equal(_np16(norms).astype(np.int64), ref16)
    else:
        assert np.array_equal(norms.cpu().numpy(), ref_norms)
    # the same codes as rpbh_quantize_weight, whose norms follow the weight's dtype
    p2, n2 = wq.rpbh_quantize_weight(_t(w, w_bf16), perm_d, signs_d, bits, cb)
    assert torch.equal(p2, packed)
    assert n2.dtype == (torch.bfloat16 if w_bf16 else torch.float32)
    if n2.dtype == ndt:
        assert torch.equal(n2, norms)


@pytest.mark.parametrize("numel", [1, 5, 7, 8, 9, 63, 1000, 12345, 3 * (1 << 20) + 5])
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_pack_unpack_codes_any_length(wq, oracle, numel, bits):
    """Page "orbit_quant.py", pack_codes / unpack_codes on flat code arrays of any length (a row
    of 5 or 7 codes starts the next row mid-byte); codes above 2^bits - 1 keep only their low bits,
    as the page's shifts and masks do. Both directions are compared byte for byte with the oracle."""
    codes = inputs.uniform_int((numel,), 256, seed=numel * 8 + bits).astype(np.uint8)
    ref = oracle.pack_codes(codes, bits)
    got = wq.rpbh_pack_codes(torch.from_numpy(codes).cuda(), bits)
    assert np.array_equal(got.cpu().numpy(), ref)
    back = wq.rpbh_unpack_codes(got, bits, numel)
    assert np.array_equal(back.cpu().numpy(), oracle.unpack_codes(ref, bits, numel))
    assert np.array_equal(back.cpu().numpy(), codes & ((1 << bits) - 1))
    # misaligned views (offset by one byte) take the byte-wise path
    buf = torch.zeros(numel + 1, dtype=torch.uint8, device="cuda")
    buf[1:] = torch.from_numpy(codes).cuda()
    got1 = wq.rpbh_pack_codes(buf[1:], bits)
    assert torch.equal(got1, got)
    out = torch.zeros(numel + 1, dtype=torch.uint8, device="cuda")
    wq.rpbh_unpack_codes(got, bits, numel, codes=out[1:])
    assert torch.equal(out[1:], back) and int(out[0]) == 0


def test_pack_codes_of_rows_with_cross_byte_offsets(wq, oracle):
    """Codes of a [rows, d] array with d not a multiple of 8 (d = 13, 3 bits: 39 bits per row), packed
    as one stream, then a row read back alone by unpacking the stream and slicing."""
    rows, d, bits = 77, 13, 3
    codes = inputs.uniform_int((rows, d), 8, seed=13).astype(np.uint8)
    got = wq.rpbh_pack_codes(torch.from_numpy(codes).cuda(), bits)
    assert np.array_equal(got.cpu().numpy(), oracle.pack_codes(codes, bits))
    back = wq.rpbh_unpack_codes(got, bits, rows * d).view(rows, d)
    assert np.array_equal(back.cpu().numpy(), codes)


def test_pack_codes_errors(wq):
    from weight_quantization_b200.ops import WQError
    c = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(WQError):
        wq.rpbh_pack_codes(c, 9)
    with pytest.raises(WQError):
        wq.rpbh_unpack_codes(torch.zeros(16, dtype=torch.uint8, device="cuda"), 0, 16)
    assert wq.rpbh_pack_codes(c[:0], 3).numel() == 0
