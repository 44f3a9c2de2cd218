"""GPU TQ3 codec on a pool of 56-byte records read and written through indirection
(tq3_encode_slots, tq3_decode_paged), through the C ABI.

The records are those of tq3_encode_aos (packed bytes, norm, scale; page "tq3_core.py",
tq3_memory_bytes' 56 bytes per vector). Scatter-encode must put, at each named slot, exactly the
record the contiguous encoder writes for that vector and leave every other record alone; paged
decode must equal the oracle's decode of the records the page table names, bit for bit, with the
record of logical vector p at table[p // page_size] * page_size + p % page_size.
"""
import numpy as np
import pytest
import torch

from weight_quantization_b200 import inputs

pytestmark = pytest.mark.gpu

SENTINEL = 0xA5
POOL_FAULT = 64


@pytest.fixture(scope="module")
def wq():
    from weight_quantization_b200 import build, ops
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ops.device_fault()  # start from clear flags
    return ops


def _x(n, seed, bf16):
    x = torch.from_numpy(inputs.gaussian((n, 128), seed=seed).astype(np.float32)).cuda()
    return x.to(torch.bfloat16) if bf16 else x


@pytest.mark.parametrize("n", [1, 257, 40001, 131072])
@pytest.mark.parametrize("bf16", [True, False])
def test_encode_slots_scatter(wq, n, bf16):
    mask = wq.sign_mask_words(inputs.tq3_sign_bits())
    x = _x(n, 10 + n, bf16)
    n_pool = 2 * n + 13
    rng = np.random.default_rng(n)
    slots = rng.permutation(n_pool)[:n].astype(np.int64)
    skip = rng.random(n) < 0.05  # padding vectors, not stored
    slots[skip] = -1
    pool = torch.full((n_pool, 56), SENTINEL, dtype=torch.uint8, device="cuda")
    wq.tq3_encode_slots(x, mask, torch.from_numpy(slots).cuda(), pool)
    want = wq.tq3_encode_aos(x, mask).reshape(n, 56).cpu().numpy()
    got = pool.cpu().numpy()
    assert wq.device_fault() == 0
    kept = slots >= 0
    assert np.array_equal(got[slots[kept]], want[kept])
    untouched = np.ones(n_pool, bool)
    untouched[slots[kept]] = False
    assert (got[untouched] == SENTINEL).all()


def test_encode_slots_outside_pool_are_skipped_and_flagged(wq):
    mask = wq.sign_mask_words(inputs.tq3_sign_bits())
    n, n_pool = 300, 400
    x = _x(n, 7, True)
    slots = np.arange(n, dtype=np.int64) + 50
    slots[[3, 100, 299]] = [n_pool, n_pool + 5, 1 << 40]
    pool = torch.full((n_pool, 56), SENTINEL, dtype=torch.uint8, device="cuda")
    wq.tq3_encode_slots(x, mask, torch.from_numpy(slots).cuda(), pool)
    want = wq.tq3_encode_aos(x, mask).reshape(n, 56).cpu().numpy()
    got = pool.cpu().numpy()
    assert wq.device_fault() == POOL_FAULT
    assert wq.device_fault() == 0  # read and cleared
    ok = slots < n_pool
    assert np.array_equal(got[slots[ok]], want[ok])
    untouched = np.ones(n_pool, bool)
    untouched[slots[ok]] = False
    assert (got[untouched] == SENTINEL).all()


def _pool_from_oracle(oracle, n_pool, seed):
    bits = inputs.tq3_sign_bits()
    x = inputs.gaussian((n_pool, 128), seed=seed).astype(np.float32)
    p, nr, sc = oracle.tq3_encode(x, bits)
    return p, nr, sc, oracle.tq3_to_records(p, nr, sc)


def _records_of(table, page_size, n_vec):
    pos = np.arange(n_vec, dtype=np.int64)
    return table[pos // page_size].astype(np.int64) * page_size + pos % page_size


@pytest.mark.parametrize("page_size,n_pages_pool,n_vec", [(1, 500, 333), (4, 300, 4 * 250 + 3), (8, 200, 8 * 150 + 6),
                                                          (16, 97, 16 * 60 + 7), (32, 64, 32 * 40),
                                                          (256, 40, 256 * 23 + 129), (4096, 12, 4096 * 9 + 5)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_decode_paged_bit_exact(wq, oracle, page_size, n_pages_pool, n_vec, out_dtype):
    bits = inputs.tq3_sign_bits()
    n_pool = n_pages_pool * page_size
    p, nr, sc, rec = _pool_from_oracle(oracle, n_pool, seed=page_size + n_vec)
    n_pages = -(-n_vec // page_size)
    table = np.random.default_rng(n_vec).permutation(n_pages_pool)[:n_pages].astype(np.int32)
    out = wq.tq3_decode_paged(torch.from_numpy(rec).cuda(), torch.from_numpy(table).cuda(), page_size, n_vec,
                              wq.sign_mask_words(bits), out_dtype=out_dtype)
    r = _records_of(table, page_size, n_vec)
    ref = oracle.tq3_decode(p[r], nr[r], sc[r], bits, out_bf16=out_dtype == torch.bfloat16)
    got = out.cpu()
    got = got.view(torch.int16).numpy().view(np.uint16) if out_dtype == torch.bfloat16 else got.numpy()
    assert np.array_equal(got.reshape(ref.shape), ref)
    assert wq.device_fault() == 0


def test_decode_paged_entries_outside_pool_decode_as_zeros(wq, oracle):
    bits = inputs.tq3_sign_bits()
    page_size, n_pool_pages, n_vec = 64, 20, 64 * 10
    p, nr, sc, rec = _pool_from_oracle(oracle, page_size * n_pool_pages, seed=3)
    table = np.arange(10, dtype=np.int32) + 5
    table[2], table[7] = -1, n_pool_pages  # one negative entry, one past the pool
    out = wq.tq3_decode_paged(torch.from_numpy(rec).cuda(), torch.from_numpy(table).cuda(), page_size, n_vec,
                              wq.sign_mask_words(bits)).cpu().numpy()
    assert wq.device_fault() == POOL_FAULT
    bad = np.zeros(n_vec, bool)
    bad[2 * page_size:3 * page_size] = True
    bad[7 * page_size:8 * page_size] = True
    assert (out[bad] == 0).all()
    r = _records_of(table, page_size, n_vec)[~bad]
    ref = oracle.tq3_decode(p[r], nr[r], sc[r], bits, out_bf16=False)
    assert np.array_equal(out[~bad], ref.reshape(-1, 128))


def test_append_then_read_through_pages(wq):
    """A cache filled by scatter-encode in arbitrary slot order reads back through its page table
    as the contiguous codec's output."""
    mask = wq.sign_mask_words(inputs.tq3_sign_bits())
    page_size, n_vec = 16, 16 * 75 + 3
    n_pages = -(-n_vec // page_size)
    table = np.random.default_rng(1).permutation(2 * n_pages)[:n_pages].astype(np.int32)
    slots = _records_of(table, page_size, n_vec)
    x = _x(n_vec, 99, True)
    pool = torch.zeros((2 * n_pages * page_size, 56), dtype=torch.uint8, device="cuda")
    wq.tq3_encode_slots(x, mask, torch.from_numpy(slots).cuda(), pool)
    got = wq.tq3_decode_paged(pool, torch.from_numpy(table).cuda(), page_size, n_vec, mask,
                              out_dtype=torch.bfloat16)
    want = wq.tq3_decode_aos(wq.tq3_encode_aos(x, mask), mask, out_dtype=torch.bfloat16).reshape(n_vec, 128)
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    assert wq.device_fault() == 0


def test_paged_argument_errors(wq):
    from weight_quantization_b200.ops import WQError
    mask = wq.sign_mask_words(inputs.tq3_sign_bits())
    pool = torch.zeros(64, 56, dtype=torch.uint8, device="cuda")
    table = torch.zeros(4, dtype=torch.int32, device="cuda")
    with pytest.raises(WQError):  # page size not a power of two
        wq.tq3_decode_paged(pool, table, 12, 8, mask)
    with pytest.raises(WQError):  # the table covers 4 * 16 vectors only
        wq.tq3_decode_paged(pool, table, 16, 65, mask)
    x = torch.zeros(4, 128, device="cuda")
    slots = torch.zeros(5, dtype=torch.int64, device="cuda")[1:]  # 8-byte aligned
    bad_pool = torch.zeros(64 * 56 + 4, dtype=torch.uint8, device="cuda")[4:].view(64, 56)
    with pytest.raises(WQError):  # pool only 4-byte aligned
        wq.tq3_encode_slots(x, mask, slots, bad_pool)
    assert wq.tq3_decode_paged(pool, table, 16, 0, mask).shape == (0, 128)
