"""GPU parity of the TQ3 kernels against the oracle, through the C ABI (page "tq3_core.py")."""
import numpy as np
import pytest
import torch

import parity
from weight_quantization_b200 import inputs

pytestmark = pytest.mark.gpu

BITS = inputs.tq3_sign_bits()


@pytest.fixture(scope="module")
def wq():
    from weight_quantization_b200 import build, ops
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return ops


@pytest.fixture(scope="module")
def mask(wq):
    return wq.sign_mask_words(BITS)


ENCODERS = [pytest.param(False, id="tq3_encode"), pytest.param(True, id="tq3_encode_exact")]
# tq3_encode decides on the unnormalised transform: its indices may differ from the step-by-step
# definition only inside the tie window. Coefficients within 1e-7 of a boundary are decided by
# rounding noise on either side (a constant block's exact zeros come out of the step-by-step
# rounding as +-6e-9, for instance); beyond that, differences are a few per million at most.
MAX_FAST_MISMATCH_FRACTION = 1e-5


def _encode(wq, x_np, is_bf16, mask, exact=False):
    t = torch.from_numpy(x_np.view(np.int16) if is_bf16 else x_np)
    t = t.view(torch.bfloat16) if is_bf16 else t
    p, n, s = wq.tq3_encode(t.cuda(), mask, exact=exact)
    torch.cuda.synchronize()
    return p.cpu().numpy(), n.cpu().numpy(), s.cpu().numpy()


def _tie_counts():
    """Oracle-only counts of coefficients within 1e-6 of a boundary (tests/golden/tq3_tie_counts.txt)."""
    from conftest import read_golden
    return {r[0]: (int(r[1]), int(r[2]), int(r[3])) for r in read_golden("tq3_tie_counts.txt")}


def _report(name, st):
    """Append the parity counts to the file named by WQ_PARITY_REPORT (a JSON line per workload), so
    that a run can keep them; the assertions below hold either way."""
    import json
    import os
    path = os.environ.get("WQ_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"workload": name, **st}) + "\n")


def _check_encoder(st, exact):
    """tq3_encode_exact reproduces the definition bit for bit; tq3_encode stays in the tie window
    (enforced by parity.check_tq3_encode) and mismatches rarely."""
    if exact:
        assert st["index_mismatches"] == 0 and st["bytes_equal"]
        assert st["norms_equal"] == st["vectors"] and st["scales_equal"] == st["vectors"]
    else:
        assert st["mismatches_beyond_1e-7"] <= MAX_FAST_MISMATCH_FRACTION * 128 * st["vectors"] + 2


@pytest.mark.parametrize("exact", ENCODERS)
def test_encode_roundtrip_config_fp32(wq, oracle, mask, exact):
    """4096 x 128 fp32: 4064 N(0,1) vectors and 32 constant blocks (value 1.0)."""
    x = inputs.tq3_roundtrip()
    p, n, s = _encode(wq, x, False, mask, exact)
    st = parity.check_tq3_encode(oracle, x, BITS, False, p, n, s)
    # every constant block has 11 exact-zero coefficients; they are exact ties at boundary 0.0
    vectors, window, zeros = _tie_counts()["tq3_roundtrip_fp32"]
    assert (st["vectors"], st["coeffs_in_tie_window"], st["exact_zero_coeffs"]) == (vectors, window, zeros)
    assert st["index_mismatches"] <= window  # every mismatch lies in the window (checked one by one)
    _check_encoder(st, exact)
    _report("tq3_roundtrip_fp32 " + ("tq3_encode_exact" if exact else "tq3_encode"), st)
    print("tq3 encode C1", "exact" if exact else "fast", st)


@pytest.mark.parametrize("exact", ENCODERS)
@pytest.mark.parametrize("n_vec", [1, 3, 33, 127, 128, 129, 1000, 40000])
@pytest.mark.parametrize("is_bf16", [False, True])
def test_encode_ragged(wq, oracle, mask, n_vec, is_bf16, exact):
    x = inputs.gaussian((n_vec, 128), seed=1000 + n_vec) * 4
    if is_bf16:
        x = inputs.to_bf16_bits(torch.from_numpy(x))
    p, n, s = _encode(wq, x, is_bf16, mask, exact)
    _check_encoder(parity.check_tq3_encode(oracle, x, BITS, is_bf16, p, n, s), exact)


@pytest.mark.parametrize("exact", ENCODERS)
def test_encode_degenerate_vectors(wq, oracle, mask, exact):
    rows = [np.zeros(128), np.full(128, 1.0), np.full(128, 2.5), np.full(128, -3.0),
            np.full(128, 1e-30), np.full(128, 1e30), np.eye(128)[5] * 7.0, np.eye(128)[0] * -1e-3,
            np.where(np.arange(128) % 2 == 0, 1.0, -1.0), np.linspace(-1, 1, 128),
            np.sin(np.linspace(0, 2 * np.pi, 128)), np.r_[np.zeros(127), 40.0]]
    x = np.array(rows, np.float32)
    p, n, s = _encode(wq, x, False, mask, exact)
    st = parity.check_tq3_encode(oracle, x, BITS, False, p, n, s)
    assert n[0] == np.float32(1e-8) and s[0] == np.float32(1e-8)
    assert p[0].tobytes() == bytes.fromhex("dbb66d") * 16
    _check_encoder(st, exact)


def test_encode_kv_cache_full_size(wq, oracle, mask):
    """K and V caches [8, 8, 4096, 128] bf16 = 524,288 vectors, every vector checked, with both
    encoders against one oracle pass."""
    k, v = inputs.kv_cache()
    keys = ("vectors", "index_mismatches", "mismatches_beyond_1e-7", "coeffs_in_tie_window", "norms_equal",
            "scales_equal")
    total = {e: {key: 0 for key in keys} for e in ("fast", "exact")}
    for name, t in (("K", k), ("V", v)):
        x = t.reshape(-1, 128)
        ref = oracle.tq3_encode_debug(x, BITS, is_bf16=True)
        for exact in (False, True):
            p, n, s = _encode(wq, x, True, mask, exact)
            st = parity.check_tq3_encode(oracle, x, BITS, True, p, n, s, ref=ref)
            _check_encoder(st, exact)
            for key in keys:
                total["exact" if exact else "fast"][key] += st[key]
    vectors, window, _ = _tie_counts()["kv_cache_bf16"]
    for e in ("fast", "exact"):
        assert total[e]["vectors"] == vectors and total[e]["coeffs_in_tie_window"] == window
        assert total[e]["index_mismatches"] <= window
        _report("kv_cache_bf16 " + ("tq3_encode_exact" if e == "exact" else "tq3_encode"), total[e])
    print("tq3 encode C2", total)


@pytest.mark.parametrize("out_bf16", [False, True])
def test_decode_roundtrip_config(wq, oracle, mask, out_bf16):
    x = inputs.tq3_roundtrip()
    packed, norms, scales = oracle.tq3_encode(x, BITS)
    out = wq.tq3_decode(torch.from_numpy(packed).cuda(), torch.from_numpy(norms).cuda(),
                        torch.from_numpy(scales).cuda(), mask,
                        out_dtype=torch.bfloat16 if out_bf16 else torch.float32)
    g = out.cpu()
    g = g.view(torch.int16).numpy().view(np.uint16) if out_bf16 else g.numpy()
    st = parity.check_tq3_decode(oracle, packed, norms, scales, BITS, g, out_bf16)
    assert st["bit_exact"]
    print("tq3 decode C1", out_bf16, st)


@pytest.mark.parametrize("n_vec", [1, 5, 129, 777, 60001])
@pytest.mark.parametrize("out_bf16", [False, True])
def test_decode_ragged(wq, oracle, mask, n_vec, out_bf16):
    idx = inputs.uniform_int((n_vec, 128), 8, seed=n_vec)
    packed = oracle.tq3_pack(idx)
    norms = (np.abs(inputs.gaussian((n_vec,), seed=n_vec + 1)) * 3 + 0.1).astype(np.float32)
    scales = (np.abs(inputs.gaussian((n_vec,), seed=n_vec + 2)) * 0.2 + 0.05).astype(np.float32)
    out = wq.tq3_decode(torch.from_numpy(packed).cuda(), torch.from_numpy(norms).cuda(),
                        torch.from_numpy(scales).cuda(), mask,
                        out_dtype=torch.bfloat16 if out_bf16 else torch.float32).cpu()
    out = out.view(torch.int16).numpy().view(np.uint16) if out_bf16 else out.numpy()
    st = parity.check_tq3_decode(oracle, packed, norms, scales, BITS, out, out_bf16)
    assert st["bit_exact"]


def test_decode_long_context_full_size(wq, oracle, mask):
    """1,048,576 records decoded to bf16 [1, 8, 131072, 128], every output compared with the
    oracle bit for bit (the decoder performs the page's roundings step by step)."""
    packed, norms, scales = inputs.long_context_records()
    out = wq.tq3_decode(torch.from_numpy(packed).cuda(), torch.from_numpy(norms).cuda(),
                        torch.from_numpy(scales).cuda(), mask, out_dtype=torch.bfloat16)
    g = out.cpu().view(torch.int16).numpy().view(np.uint16)
    st = parity.check_tq3_decode(oracle, packed, norms, scales, BITS, g, True)
    assert st["bit_exact"] and st["vectors"] == 1 << 20
    _report("long_context_bf16 tq3_decode", st)
    print("tq3 decode C3", st)


def test_roundtrip_quality_on_gpu(wq, mask):
    """The page's quality bar (mean cosine > 0.97) holds for the GPU round trip."""
    x = torch.from_numpy(inputs.tq3_roundtrip()).cuda()
    p, n, s = wq.tq3_encode(x, mask)
    xr = wq.tq3_decode(p, n, s, mask).reshape(x.shape)
    cos = torch.nn.functional.cosine_similarity(x.double(), xr.double(), dim=-1)
    assert cos[:4064].mean().item() > 0.97
    assert cos[4064:].min().item() > 0.97


def test_outputs_stay_in_bounds_and_streams(wq, oracle, mask):
    """Canaries after the last record stay untouched; work runs on the caller's stream."""
    n_vec = 77
    x = torch.from_numpy(inputs.gaussian((n_vec, 128), seed=9)).cuda()
    packed = torch.full((n_vec + 3, 48), 0xAB, dtype=torch.uint8, device="cuda")
    norms = torch.full((n_vec + 5,), -7.0, device="cuda")
    scales = torch.full((n_vec + 5,), -7.0, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        wq.tq3_encode(x, mask, packed=packed[:n_vec], norms=norms[:n_vec], scales=scales[:n_vec])
        out = torch.full((n_vec + 2, 128), -9.0, device="cuda")
        wq.tq3_decode(packed[:n_vec], norms[:n_vec], scales[:n_vec], mask, out=out[:n_vec])
    s.synchronize()
    assert bool((packed[n_vec:] == 0xAB).all()) and bool((norms[n_vec:] == -7).all())
    assert bool((scales[n_vec:] == -7).all()) and bool((out[n_vec:] == -9).all())
    parity.check_tq3_encode(oracle, x.cpu().numpy(), BITS, False, packed[:n_vec].cpu().numpy(),
                            norms[:n_vec].cpu().numpy(), scales[:n_vec].cpu().numpy())


def test_empty_and_errors(wq, mask):
    x = torch.empty(0, 128, device="cuda")
    p, n, s = wq.tq3_encode(x, mask)
    assert p.shape == (0, 1, 48)
    with pytest.raises(wq.WQError):
        wq.tq3_encode(torch.zeros(4, 128, device="cuda", dtype=torch.float32)[:, :128], mask,
                      packed=torch.empty(4 * 48 + 1, dtype=torch.uint8, device="cuda")[1:].view(4, 1, 48))


@pytest.mark.parametrize("exact", ENCODERS)
@pytest.mark.parametrize("table", ["seed7", "all_plus", "all_minus"])
@pytest.mark.parametrize("is_bf16", [False, True])
def test_other_sign_tables(wq, oracle, table, is_bf16, exact):
    """Sign tables other than the page's seed-42 draws take the runtime-mask kernels."""
    bits = {"seed7": inputs.tq3_sign_bits(7), "all_plus": np.ones(128, np.uint8),
            "all_minus": np.zeros(128, np.uint8)}[table]
    m = wq.sign_mask_words(bits)
    x = inputs.gaussian((300, 128), seed=77) * 3
    x[5] = 2.5  # a constant block
    x[6] = 0.0
    if is_bf16:
        x = inputs.to_bf16_bits(torch.from_numpy(x))
    t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if is_bf16 else torch.from_numpy(x)
    p, n, s = wq.tq3_encode(t.cuda(), m, exact=exact)
    st = parity.check_tq3_encode(oracle, x, bits, is_bf16, p.cpu().numpy(), n.cpu().numpy(), s.cpu().numpy())
    _check_encoder(st, exact)
    for out_dtype in (torch.float32, torch.bfloat16):
        out = wq.tq3_decode(p, n, s, m, out_dtype=out_dtype).cpu()
        g = out.view(torch.int16).numpy().view(np.uint16) if out_dtype == torch.bfloat16 else out.numpy()
        st = parity.check_tq3_decode(oracle, p.cpu().numpy().reshape(-1, 48), n.cpu().numpy().ravel(),
                                     s.cpu().numpy().ravel(), bits, g, out_dtype == torch.bfloat16)
        assert st["bit_exact"]


@pytest.mark.parametrize("exact", ENCODERS)
def test_extreme_dynamic_range(wq, oracle, mask, exact):
    """Vectors spanning many binades (down to subnormal quotients, up to squares beyond the fp32
    range): the exact encoder still matches the oracle's IEEE divisions bit for bit, the fast one
    stays inside the tie window."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((2000, 128)) * np.exp(rng.uniform(-40, 40, (2000, 128)))).astype(np.float32)
    x[:20, :64] = 1e-40  # subnormal inputs next to normal ones
    x[20:40] = np.float32(3e-39)
    x[40:60, 0] = 3e38
    p, n, s = _encode(wq, x, False, mask, exact)
    _check_encoder(parity.check_tq3_encode(oracle, x, BITS, False, p, n, s), exact)
    xb = inputs.to_bf16_bits(torch.from_numpy(x))
    p, n, s = _encode(wq, xb, True, mask, exact)
    _check_encoder(parity.check_tq3_encode(oracle, xb, BITS, True, p, n, s), exact)


def _overflow_rows():
    """Finite vectors whose unnormalised Hadamard coefficients leave the fp32 range (sum |x| above
    FLT_MAX), next to vectors just below and above the size where the fp32 sum of squares
    overflows. The page normalises before transforming (tq3_quantize steps 1-3), so every one of
    them has an ordinary encoding."""
    rng = np.random.default_rng(17)
    rows = [np.full(128, 1e37), np.full(128, -3e37), np.full(128, 3e38),
            np.r_[2e38, np.zeros(50), 2e38, np.zeros(76)], np.r_[-2e38, -2e38, rng.standard_normal(126)],
            np.full(128, 1.5e36), np.where(np.arange(128) % 3 == 0, 3e38, -1e38)]
    g = rng.standard_normal((40, 128))
    rows += list(g[:10] * 1e36) + list(g[10:20] * 1.5e18) + list(g[20:30] * 3e18) + list(g[30:] * 1e19)
    mixed = rng.standard_normal((30, 128)) * np.exp(rng.uniform(0, 87, (30, 128)))  # up to ~6e37
    rows += list(mixed)
    return np.array(rows, np.float32)


@pytest.mark.parametrize("exact", ENCODERS)
@pytest.mark.parametrize("is_bf16", [False, True])
def test_encode_beyond_fp32_transform(wq, oracle, mask, is_bf16, exact):
    """Constant blocks of 1e37 and -3e37, all entries at 3e38 (norm beyond fp32: +inf, all indices
    3), two entries of 2e38 of one sign, and random vectors up to 6e37: element by element
    against the oracle, with the tie window, in every record layout the encoders write."""
    x = _overflow_rows()
    if is_bf16:
        x = inputs.to_bf16_bits(torch.from_numpy(x))
    p, n, s = _encode(wq, x, is_bf16, mask, exact)
    st = parity.check_tq3_encode(oracle, x, BITS, is_bf16, p, n, s)
    _check_encoder(st, exact)
    assert np.isinf(n[2]) and p[2].tobytes() == bytes.fromhex("dbb66d") * 16
    if exact:
        return
    t = torch.from_numpy(x.view(np.int16) if is_bf16 else x)
    t = (t.view(torch.bfloat16) if is_bf16 else t).cuda()
    rec = wq.tq3_encode_aos(t, mask)
    pool = torch.zeros(2 * len(x), 56, dtype=torch.uint8, device="cuda")
    slots = torch.arange(len(x), dtype=torch.int64, device="cuda") * 2 + 1
    wq.tq3_encode_slots(t, mask, slots, pool)
    torch.cuda.synchronize()
    want = np.concatenate([p.reshape(-1, 48), n.reshape(-1, 1).view(np.uint8), s.reshape(-1, 1).view(np.uint8)],
                          axis=1)
    assert np.array_equal(rec.cpu().numpy().reshape(-1, 56), want)
    assert np.array_equal(pool.cpu().numpy()[1::2], want)
    assert not pool.cpu().numpy()[0::2].any()


def test_no_device_fault_recorded(wq):
    torch.cuda.synchronize()
    assert wq.device_fault() == 0
