"""Host checks of the address arithmetic behind the library's bulk copies and L2 prefetches that
depend on the call's shapes. A bulk copy or prefetch must start on a 16-byte boundary and move a
multiple of 16 bytes; these tests restate, in Python, how the kernels form each range and check
those rules, the bounds of the buffer and which records a range holds, for every launch shape the
GPU tests use and more. The GPU tests run the kernels themselves.

* Paged TQ3 decode (page "tq3_core.py", the 56-byte records of tq3_memory_bytes read through a page
  table): the records of the tile two rounds ahead are prefetched page by page, lane l taking page
  l for pages of 4 to 16 records, lane 0 the one page for pages of 32 or more.
* Attention over a contiguous TQ3 cache: a whole tile of kKeys records of head h, keys
  t kKeys .. (t + 1) kKeys - 1, is one bulk copy when h S is even.
"""
import random

import pytest

TILE = 32  # vectors per decoder tile


def paged_prefetches(page_size, n_pool, n_vec, grid, table):
    """Every (lane, record range) the paged decoder prefetches, in the kernel's arithmetic."""
    shift = page_size.bit_length() - 1
    n_tiles = -(-n_vec // TILE)
    pf_lanes = 1 if shift >= 5 else (TILE >> shift) if shift >= 2 else 0
    out = []
    for tid in range(TILE):
        def page_entry(t):
            first = 0 if shift >= 5 else tid << shift
            if tid < pf_lanes and t < n_tiles and t * TILE + first < n_vec:
                idx = (t * TILE + first) >> shift
                assert 0 <= idx < len(table), "page-table read out of range"
                return table[idx]
            return -1
        for block in range(grid):
            tile = block
            pe = page_entry(tile + 2 * grid)
            while tile < n_tiles:
                pe_next = page_entry(tile + 3 * grid)
                if pe >= 0:
                    v0 = (tile + 2 * grid) * TILE
                    cnt = min(n_vec - v0, TILE) & ~3
                    first = 0 if shift >= 5 else tid << shift
                    per = TILE if shift >= 5 else 1 << shift
                    c = min(cnt - first, per)
                    lp = v0 + first
                    r0 = (pe << shift) | (lp & ((1 << shift) - 1))
                    if c > 0 and r0 + c <= n_pool:
                        out.append((lp, r0, c))
                pe = pe_next
                tile += grid
    return out


@pytest.mark.parametrize("page_size,n_pool_pages,n_vec", [
    (1, 500, 333), (2, 400, 700), (4, 300, 4 * 250 + 3), (8, 200, 8 * 150 + 6), (16, 97, 16 * 60 + 7),
    (32, 64, 32 * 40), (256, 40, 256 * 23 + 129), (4096, 12, 4096 * 9 + 5)])
@pytest.mark.parametrize("grid", [1, 2, 3, 7, 1776])
def test_paged_decode_prefetch_ranges(page_size, n_pool_pages, n_vec, grid):
    rng = random.Random(page_size * 7919 + n_vec)
    n_pool = n_pool_pages * page_size
    table = [rng.randrange(-1, n_pool_pages) for _ in range(-(-n_vec // page_size))]
    grid = min(grid, -(-n_vec // TILE))
    base = 1 << 20  # a 16-byte-aligned pool (the kernel prefetches only from one)
    for lp, r0, c in paged_prefetches(page_size, n_pool, n_vec, grid, table):
        assert (base + 56 * r0) % 16 == 0 and (56 * c) % 16 == 0
        assert 0 <= r0 and r0 + c <= n_pool
        for i in range(c):  # the range holds exactly the records of the tile's vectors lp .. lp + c - 1
            p = lp + i
            assert table[p // page_size] * page_size + p % page_size == r0 + i


@pytest.mark.parametrize("keys_per_tile", [128, 256])
@pytest.mark.parametrize("heads,S", [(64, 32768), (3, 4097), (5, 129), (2, 256), (7, 1000), (1, 1)])
def test_attention_bulk_tile_ranges(keys_per_tile, heads, S):
    base = 1 << 20
    tile_bytes = 56 * keys_per_tile
    assert tile_bytes % 16 == 0
    for h in range(heads):
        bulk_ok = (h * S) % 2 == 0
        for t in range(-(-S // keys_per_tile)):
            if not (bulk_ok and (t + 1) * keys_per_tile <= S):
                continue  # per-thread copies
            first = h * S + t * keys_per_tile
            assert (base + 56 * first) % 16 == 0
            assert h * S <= first and first + keys_per_tile <= (h + 1) * S  # inside head h
