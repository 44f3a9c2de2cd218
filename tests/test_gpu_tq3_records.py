"""GPU TQ3 codec on 56-byte records (tq3_encode_aos, tq3_decode_aos), through the C ABI: the same
arithmetic as the three-array forms, so encode equals their interleaved output byte for byte and
decode equals the oracle bit for bit."""
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


@pytest.mark.parametrize("n", [1, 257, 40001, 131072])
@pytest.mark.parametrize("bf16", [True, False])
def test_encode_records_equal_three_arrays(wq, oracle, n, bf16):
    bits = inputs.tq3_sign_bits()
    mask = wq.sign_mask_words(bits)
    x = torch.from_numpy(inputs.gaussian((n, 128), seed=n).astype(np.float32)).cuda()
    if bf16:
        x = x.to(torch.bfloat16)
    rec = wq.tq3_encode_aos(x, mask)
    p, nr, sc = wq.tq3_encode(x, mask)
    ref = oracle.tq3_to_records(p.cpu().numpy(), nr.cpu().numpy(), sc.cpu().numpy())
    assert rec.shape == (n, 1, 56)
    assert np.array_equal(rec.cpu().numpy().reshape(n, 56), ref)


@pytest.mark.parametrize("n", [1, 300, 70001])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_decode_records_bit_exact(wq, oracle, n, out_dtype):
    bits = inputs.tq3_sign_bits()
    x = inputs.gaussian((n, 128), seed=n + 1).astype(np.float32)
    p, nr, sc = oracle.tq3_encode(x, bits)
    rec = torch.from_numpy(oracle.tq3_to_records(p, nr, sc)).cuda()
    out = wq.tq3_decode_aos(rec, wq.sign_mask_words(bits), out_dtype=out_dtype)
    ref = oracle.tq3_decode(p, nr, sc, bits, out_bf16=out_dtype == torch.bfloat16)
    got = out.cpu()
    got = got.view(torch.int16).numpy().view(np.uint16) if out_dtype == torch.bfloat16 else got.numpy()
    assert np.array_equal(got.reshape(ref.shape), ref)
    assert wq.device_fault() == 0


def test_records_argument_errors(wq):
    from weight_quantization_b200.ops import WQError
    x = torch.zeros(4, 128, device="cuda")
    rec = torch.zeros(4 * 56 + 4, dtype=torch.uint8, device="cuda")[4:].view(4, 56)  # 4-byte aligned only
    with pytest.raises(WQError):
        wq.tq3_encode_aos(x, wq.sign_mask_words(inputs.tq3_sign_bits()), records=rec)
