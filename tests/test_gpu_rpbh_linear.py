"""GPU parity of the fused RPBH linear layer (page "orbit_quant.py", forward: F.linear of the rotated
activations with the rotated-basis weight) against the oracle, through the C ABI.

Tolerance, from the arithmetic: the kernel scales the fp32 sum by the row norm instead of rounding
each bf16 product bf16(codebook) * bf16(norm) to bf16 (at most 2^-8 relative per term), sums in
fp32 in its own order (at most d * 2^-24 relative to sum |terms| per term, doubled for safety) and
rounds y once to bf16 (2^-8 relative; 2^-7 allowed). So |y - y_ref| <= (2^-8 + d 2^-23) A + 2^-7 |y_ref|
with A = sum_k |x_rot W'| from the oracle.
"""
import numpy as np
import pytest
import torch

from weight_quantization_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wq():
    from weight_quantization_b200 import build, ops
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return ops


def _bf16_dev(bits16):
    return torch.from_numpy(np.ascontiguousarray(bits16).view(np.int16)).view(torch.bfloat16).cuda()


def _case(wq, oracle, out_f, d, m, bits, norm_bf16, with_bias, seed, check_rows=None):
    cb = oracle.rpbh_codebook(bits, d)
    codes = inputs.uniform_int((out_f, d), 1 << bits, seed=seed)
    packed = oracle.pack_codes(codes, bits)
    norms32 = (np.abs(inputs.gaussian((out_f,), seed=seed + 1)) * 0.7 + 0.05).astype(np.float32)
    if norm_bf16:
        n16 = oracle.f32_array_to_bf16(norms32)
        norms_dev, norms_f32 = _bf16_dev(n16), oracle.bf16_array_to_f32(n16)
    else:
        norms_dev, norms_f32 = torch.from_numpy(norms32).cuda(), norms32
    x = oracle.f32_array_to_bf16(inputs.gaussian((m, d), seed=seed + 2).astype(np.float32))
    bias = None
    if with_bias:
        bias = oracle.f32_array_to_bf16((inputs.gaussian((out_f,), seed=seed + 3) * 0.1).astype(np.float32))
    y = wq.rpbh_linear(torch.from_numpy(packed).cuda(), norms_dev, out_f, d, bits, cb, _bf16_dev(x),
                       bias=_bf16_dev(bias) if bias is not None else None)
    torch.cuda.synchronize()
    assert wq.device_fault() == 0
    got = oracle.bf16_array_to_f32(y.cpu().view(torch.int16).numpy().view(np.uint16)).astype(np.float64)
    rows = np.arange(m) if check_rows is None else np.asarray(check_rows)
    ref, a = oracle.rpbh_linear(packed, norms_f32, out_f, d, bits, cb, x[rows], bias)
    tol = (2.0 ** -8 + d * 2.0 ** -23) * a + 2.0 ** -7 * np.abs(ref) + 1e-30
    err = np.abs(got[rows] - ref)
    worst = float((err / tol).max())
    assert worst <= 1.0, f"worst error {worst:.3f} of the tolerance"
    return worst


@pytest.mark.parametrize("out_f,d,m", [(128, 64, 256), (300, 192, 100), (256, 512, 513), (1, 64, 1), (130, 1024, 257)])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_linear_small(wq, oracle, out_f, d, m, bits):
    _case(wq, oracle, out_f, d, m, bits, norm_bf16=True, with_bias=True, seed=out_f + d + m + bits)


@pytest.mark.parametrize("norm_bf16,with_bias", [(False, True), (True, False), (False, False)])
def test_linear_norm_dtype_and_bias(wq, oracle, norm_bf16, with_bias):
    _case(wq, oracle, 200, 320, 300, 3, norm_bf16=norm_bf16, with_bias=with_bias, seed=11)


def test_linear_llm_full_size_sampled_rows(wq, oracle):
    """W[4096, 11008] at 3 bits times x_rot[2048, 11008]: every output of 264 activation rows (every
    eighth row, which touches each of the kernel's 256-row tiles 32 times, plus the first and last
    rows of every tile), against the fp64 oracle."""
    rows = np.unique(np.concatenate([np.arange(0, 2048, 8), np.arange(0, 2048, 256) + 255]))
    _case(wq, oracle, 4096, 11008, 2048, 3, norm_bf16=True, with_bias=True, seed=42, check_rows=rows)


def test_linear_errors(wq):
    from weight_quantization_b200.ops import WQError
    packed = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    norms = torch.ones(8, dtype=torch.bfloat16, device="cuda")
    x = torch.zeros(4, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(WQError):  # d not a multiple of 64
        wq.rpbh_linear(packed, norms, 8, 96, 3, np.linspace(-1, 1, 8, dtype=np.float32), x)
    with pytest.raises(WQError):  # bits
        wq.rpbh_linear(packed, norms, 8, 64, 5, np.linspace(-1, 1, 32, dtype=np.float32), x[:, :64].contiguous())
    y = wq.rpbh_linear(packed, norms, 8, 64, 3, np.linspace(-1, 1, 8, dtype=np.float32), x[:0, :64].contiguous())
    assert y.shape == (0, 8)
