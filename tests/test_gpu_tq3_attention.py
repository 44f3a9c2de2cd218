"""GPU attention over a TQ3-compressed K/V cache (tq3_attention) against the oracle, through the C ABI.

The oracle decodes every key and value with the page's tq3_dequantize (page "tq3_core.py") and takes
softmax(softmax_scale q k^T) v in fp64. The kernel never decodes: it rotates q into the indices'
basis, scores and accumulates there in fp32, and rotates each output row back once.

Tolerance, from the arithmetic (u = 2^-24, first order):
* logits. The kernel's logit for key j is a 128-term fp32 dot product of the rotated query (seven
  rounded butterfly stages) with the key's centroids, times norm * scale * post * softmax_scale * log2 e.
  Bounding each rounding by u times the sum of absolute terms, and that sum by Cauchy-Schwarz, gives
  |d logit_j| <= (128 + 7 sqrt(128) + 10) u * softmax_scale |q| |k_j| < 2^-16 softmax_scale |q| max_j |k_j|
  =: L (the last 10 u cover the page's own rounding of k_j, the coefficient and the max subtraction).
* weights. Logits off by at most L change every normalised weight by a factor within e^(+-2L), so
  the output moves by at most (e^(4L) - 1) max_j |v_j|_inf <= 4.4 L max_j |v_j|_inf; exp2f adds
  2^-21 max_j |v_j|_inf.
* values. Each rotated accumulator sums at most n = ceil(S / splits) + 8 weighted centroids in fp32
  (the running sum over this CTA's keys, then the cluster merge) and is rescaled once per tile of
  128 or 256 keys; with splits counted for 256-key tiles (the fewest) and one rounding per tile
  added, n = ceil(S / splits) + ceil(S / 128) + 8. The inverse transform adds seven stages; bounded
  as above this is (n + 40) u max_j |v_j|_2 on every output element.
* bf16 output: one rounding, 2^-8 |out| allowed.

From 48 query rows per head on, the call takes the tensor-core path: the products run on bf16
operands, each fp32 operand split into hi + lo (residual at most 2^-18 of the value) and three
passes hi hi + hi lo + lo hi accumulated in fp32. Per product term that adds 3 * 2^-18 (two split
residuals and the dropped lo lo) and one rounding of the folded key or value factor, and each
128-key tile accumulates 3 * 128 = 384 terms; so there
* logits: |d logit_j| <= (3 * 2^-18 + (384 + 7 sqrt(128) + 12) u) softmax_scale |q| |k_j|, below
  2^-14 softmax_scale |q| max_j |k_j| =: L_tc, and the weights move as above with L_tc for L;
* values: (3 * 2^-18 + (384 + ceil(S / 128) + 48) u) max_j |v_j|_2 on every output element (the
  tile products, the per-tile accumulation in tensor memory and the rare rescales of the running
  max).
"""

MMA_MIN_ROWS = 48
import math

import numpy as np
import pytest
import torch

from weight_quantization_b200 import inputs

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


@pytest.fixture(scope="module")
def wq():
    from weight_quantization_b200 import build, ops
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return ops


def _cache(oracle, heads, S, seed):
    """Records of a K and a V cache: Gaussian vectors with a per-token offset, as in the KV recipe."""
    bits = inputs.tq3_sign_bits()
    recs, dec = [], []
    for i in range(2):
        x = inputs.gaussian((heads * S, 128), seed=seed + i).astype(np.float32)
        x += 2.0 * inputs.gaussian((heads * S, 1), seed=seed + 10 + i).astype(np.float32)
        r = oracle.tq3_to_records(*oracle.tq3_encode(x, bits))
        recs.append(r.reshape(heads, S, 56))
        dec.append(oracle.tq3_decode(*oracle.tq3_from_records(r), bits).astype(np.float64).reshape(heads, S, 128))
    return bits, recs, dec


def _tolerance(qf, k, v, S, scale, ref, out_bf16):
    m = qf.shape[1]
    vinf = np.abs(v).max(axis=(1, 2))                   # per head
    v2 = np.linalg.norm(v, axis=2).max(axis=1)
    k2 = np.linalg.norm(k, axis=2).max(axis=1)
    qn = np.linalg.norm(qf.astype(np.float64), axis=2)
    if m >= MMA_MIN_ROWS:                               # tensor-core path
        L = 2.0 ** -14 * scale * qn * k2[:, None]
        eps = 3 * 2.0 ** -18 + (384 + -(-S // 128) + 48) * U
    else:
        splits = min(8, -(-S // 256))
        n = -(-S // splits) + -(-S // 128) + 8
        L = 2.0 ** -16 * scale * qn * k2[:, None]      # [heads, m]
        eps = (n + 40) * U
    tol = (4.4 * L + 2.0 ** -21)[:, :, None] * vinf[:, None, None] + (eps * v2)[:, None, None]
    if out_bf16:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    return tol


def _check(wq, oracle, heads, m, S, q_bf16, out_bf16, scale, seed):
    bits, (kr, vr), (k, v) = _cache(oracle, heads, S, seed)
    qf = (inputs.gaussian((heads, m, 128), seed=seed + 5) * 1.5).astype(np.float32)
    if q_bf16:
        qb = oracle.f32_array_to_bf16(qf)
        qf = oracle.bf16_array_to_f32(qb).reshape(heads, m, 128)
        q_dev = torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).cuda()
    else:
        q_dev = torch.from_numpy(qf).cuda()
    out = wq.tq3_attention(q_dev, torch.from_numpy(kr).cuda(), torch.from_numpy(vr).cuda(), wq.sign_mask_words(bits),
                           softmax_scale=scale, out_dtype=torch.bfloat16 if out_bf16 else torch.float32)
    torch.cuda.synchronize()
    if out_bf16:
        got = oracle.bf16_array_to_f32(out.cpu().view(torch.int16).numpy().view(np.uint16)).astype(np.float64)
    else:
        got = out.cpu().numpy().astype(np.float64)
    ref = oracle.tq3_attention(qf, kr, vr, bits, scale)
    tol = _tolerance(qf, k, v, S, scale, ref, out_bf16)
    err = np.abs(got - ref)
    worst = float((err / tol).max())
    assert worst <= 1.0, f"worst error {worst:.3f} of the tolerance (max abs err {err.max():.3g})"
    return worst


@pytest.mark.parametrize("heads,m,S", [(1, 1, 1), (3, 4, 127), (2, 8, 1000), (5, 16, 4097), (2, 3, 128 * 8 * 3 + 5),
                                       (4, 2, 129), (2, 17, 700), (2, 32, 2049), (1, 128, 1500), (3, 40, 256),
                                       (2, 48, 129), (3, 64, 1000), (2, 130, 300), (1, 256, 4096)])
@pytest.mark.parametrize("q_bf16", [True, False])
def test_attention_matches_oracle(wq, oracle, heads, m, S, q_bf16):
    _check(wq, oracle, heads, m, S, q_bf16, False, 128 ** -0.5, seed=heads * 1000 + m * 10 + S)


@pytest.mark.parametrize("m", [1, 5, 8])
def test_attention_bf16_out_and_sharp_softmax(wq, oracle, m):
    _check(wq, oracle, 3, m, 2000, True, True, 0.5, seed=7 + m)


def test_attention_long_context(wq, oracle):
    """32768 keys per head: the full cluster split, long per-CTA accumulations."""
    _check(wq, oracle, 2, 8, 32768, True, False, 128 ** -0.5, seed=31)


def test_attention_argument_errors(wq):
    from weight_quantization_b200.ops import WQError
    mask = wq.sign_mask_words(inputs.tq3_sign_bits())
    rec = torch.zeros(2, 16, 56, dtype=torch.uint8, device="cuda")
    with pytest.raises(WQError):  # no keys
        empty = torch.zeros(2, 0, 56, dtype=torch.uint8, device="cuda")
        wq.tq3_attention(torch.zeros(2, 1, 128, device="cuda"), empty, empty, mask)
    with pytest.raises(WQError):
        wq.tq3_attention(torch.zeros(2, 1, 128, device="cuda"), rec, rec, mask, softmax_scale=math.inf)
    assert wq.tq3_attention(torch.zeros(0, 1, 128, device="cuda"), rec[:0], rec[:0], mask).shape == (0, 1, 128)


@pytest.mark.parametrize("heads,m,S,page_size", [(3, 4, 1000, 16), (2, 8, 4097, 128), (2, 1, 300, 1), (1, 20, 777, 64),
                                                  (2, 128, 1000, 32)])
def test_attention_paged_matches_oracle(wq, oracle, heads, m, S, page_size):
    """tq3_attention_paged: the heads' pages scattered in random order over a pool (with unused
    records between them), against the oracle on the records gathered back into order."""
    bits, (kr, vr), (k, v) = _cache(oracle, heads, S, seed=500 + m + page_size)
    pph = -(-S // page_size) + 1                         # one spare page-table entry per head
    n_pages = heads * pph + 5
    order = np.random.default_rng(S).permutation(n_pages)
    table = order[:heads * pph].reshape(heads, pph).astype(np.int32)
    kpool = np.zeros((n_pages * page_size, 56), np.uint8)
    vpool = np.zeros_like(kpool)
    for h in range(heads):
        for j in range(S):
            rec = table[h, j // page_size] * page_size + j % page_size
            kpool[rec], vpool[rec] = kr[h, j], vr[h, j]
    qf = (inputs.gaussian((heads, m, 128), seed=S + 3) * 1.5).astype(np.float32)
    out = wq.tq3_attention_paged(torch.from_numpy(qf).cuda(), torch.from_numpy(kpool).cuda(),
                                 torch.from_numpy(vpool).cuda(), torch.from_numpy(table).cuda(), page_size, S,
                                 wq.sign_mask_words(bits))
    torch.cuda.synchronize()
    assert wq.device_fault() == 0
    got = out.cpu().numpy().astype(np.float64)
    ref = oracle.tq3_attention(qf, kr, vr, bits, 128 ** -0.5)
    tol = _tolerance(qf, k, v, S, 128 ** -0.5, ref, False)
    assert float((np.abs(got - ref) / tol).max()) <= 1.0
    # the contiguous call on the same records agrees to the same tolerance
    out2 = wq.tq3_attention(torch.from_numpy(qf).cuda(), torch.from_numpy(kr).cuda(), torch.from_numpy(vr).cuda(),
                            wq.sign_mask_words(bits)).cpu().numpy().astype(np.float64)
    assert float((np.abs(out2 - ref) / tol).max()) <= 1.0


def test_attention_paged_masks_entries_outside_the_pool(wq, oracle):
    """A page-table entry outside the pool masks its keys out and raises fault bit 6; the rest of the
    head attends over the remaining keys."""
    heads, m, S, ps = 1, 4, 64, 16
    bits, (kr, vr), _ = _cache(oracle, heads, S, seed=77)
    kpool, vpool = kr.reshape(S, 56).copy(), vr.reshape(S, 56).copy()
    table = np.array([[0, 1, 99, 3]], np.int32)          # page 2 points past the 4-page pool
    qf = (inputs.gaussian((heads, m, 128), seed=78)).astype(np.float32)
    wq.device_fault()
    out = wq.tq3_attention_paged(torch.from_numpy(qf).cuda(), torch.from_numpy(kpool).cuda(),
                                 torch.from_numpy(vpool).cuda(), torch.from_numpy(table).cuda(), ps, S,
                                 wq.sign_mask_words(bits))
    torch.cuda.synchronize()
    assert wq.device_fault() & 64
    keep = np.r_[np.arange(0, 32), np.arange(48, 64)]
    ref = oracle.tq3_attention(qf, kr[:, keep], vr[:, keep], bits, 128 ** -0.5)
    assert np.allclose(out.cpu().numpy(), ref, rtol=0, atol=1e-4 * np.abs(ref).max())
