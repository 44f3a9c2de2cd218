"""The device fault path, exercised without a GPU fault: a bounded wait that runs out sets a fault
bit, the host reads and clears it, and the context keeps working."""
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


def test_bounded_wait_timeout_reports_and_recovers(wq, oracle):
    wq.device_fault()  # start from clear flags
    wq.selftest_wait_timeout()
    torch.cuda.synchronize()
    assert wq.device_fault() == 32  # bit 5: the self-test's wait gave up
    assert wq.device_fault() == 0   # read-and-clear
    # the context is intact: a TQ3 encode right after still matches the oracle bit for bit
    x = inputs.gaussian((256, 128), seed=9).astype(np.float32)
    bits = inputs.tq3_sign_bits()
    p, n, s = wq.tq3_encode(torch.from_numpy(x).cuda(), wq.sign_mask_words(bits), exact=True)
    rp, rn, rs = oracle.tq3_encode(x, bits)
    assert np.array_equal(p.cpu().numpy().reshape(rp.shape), rp)
    assert np.array_equal(n.cpu().numpy().reshape(rn.shape), rn)
    assert wq.device_fault() == 0
