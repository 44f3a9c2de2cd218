"""Host check of the codebook lookup that the fused linear layer's unpacking warps use for 2- and
3-bit codes (page "orbit_quant.py": pack_codes / unpack_codes, MSB-first code stream, and
_dequantize_rotated's codebook[codes]).

The kernel never indexes a table in memory. It keeps the low and high bytes of the 2^bits bf16
codebook entries as two 8-byte tables, spreads four codes into the nibbles of a byte-permute
selector with two multiply-adds, and lets byte permutes fetch and interleave the bytes. This test
emulates those steps bit for bit (the permute's byte selection, the multiply-adds modulo 2^32, the
selector constants) and checks them against the oracle's unpacking of the same bytes, for every
possible group of eight codes, so that a wrong shift, mask or selector in the scheme shows up
without a GPU. The GPU parity tests check the kernel itself.
"""
import numpy as np
import pytest

M32 = 0xFFFFFFFF


def prmt(a, b, sel):
    """Byte permute, default mode: byte k of the result is byte (nibble k of sel) of the eight bytes
    a (bytes 0-3) then b (bytes 4-7). The scheme never sets a nibble's top bit."""
    src = [(a >> (8 * i)) & 255 for i in range(4)] + [(b >> (8 * i)) & 255 for i in range(4)]
    out = 0
    for k in range(4):
        n = (sel >> (4 * k)) & 15
        assert n < 8, "a selector nibble with its top bit set would replicate a sign"
        out |= src[n] << (8 * k)
    return out


def spread4(x, bits):
    """Four bits-wide codes of x (first code in the top bits) into selector nibbles, last code in
    nibble 0: two exact multiply-adds, as the kernel computes them."""
    if bits == 3:
        y = ((x & 0xFC0) * 3 + x) & M32
        return ((y & 0x3838) + y) & M32
    y = ((x & 0xF0) * 15 + x) & M32
    return ((y & 0x0C0C) * 3 + y) & M32


def tables(entries, bits):
    lo = [e & 255 for e in entries] + [0] * (8 - len(entries))
    hi = [e >> 8 for e in entries] + [0] * (8 - len(entries))
    word = lambda v: sum(v[k] << (8 * k) for k in range(4))
    return word(lo[:4]), word(lo[4:]), word(hi[:4]), word(hi[4:])


def lookup_chunk(raw, bits, entries):
    """One 64-code chunk (8 * bits stream bytes) to 32 bf16 pairs, code 2u in the low half of word u."""
    R = [int.from_bytes(bytes(raw[4 * i:4 * i + 4]), "little") for i in range(2 * bits)]
    lo0, lo1, hi0, hi1 = tables(entries, bits)
    words = []
    for j in range(8):
        if bits == 3:
            b0 = 3 * j
            q, u = b0 >> 2, b0 & 3
            g = prmt(R[q], R[q + 1] if q + 1 < 2 * bits else 0, (u + 2) | ((u + 1) << 4) | (u << 8))
            xa, xb = (g >> 12) & 0xFFF, g & 0xFFF
        else:
            b0 = 2 * j
            q, u = b0 >> 2, b0 & 3
            g = prmt(R[q], 0, (u + 1) | (u << 4))
            xa, xb = (g >> 8) & 0xFF, g & 0xFF
        for x in (xa, xb):
            sel = spread4(x, bits)
            L, H = prmt(lo0, lo1, sel), prmt(hi0, hi1, sel)
            words += [prmt(L, H, 0x6273), prmt(L, H, 0x4051)]
    return words


@pytest.mark.parametrize("bits", [2, 3])
def test_every_code_group_against_the_oracle_unpacking(oracle, bits):
    # every value of a group of eight codes (one byte per four 2-bit codes, three bytes per eight
    # 3-bit codes) in each of the eight positions of a chunk, with distinct entries per code
    rng = np.random.default_rng(bits)
    entries = [int(v) for v in rng.choice(1 << 16, size=1 << bits, replace=False)]
    group_bytes = bits  # eight codes of `bits` bits
    if bits == 2:
        groups = [v.to_bytes(2, "big") for v in range(1 << 16)]  # every group of eight 2-bit codes
    else:
        # each 24-bit group is two independent 12-bit halves; cover all 4096 values of each half
        groups = [((a << 12) | (a ^ 0xA5A)).to_bytes(3, "big") for a in range(4096)]
        groups += [(((b * 2654435761) & 0xFFF) << 12 | b).to_bytes(3, "big") for b in range(4096)]
    for start in range(0, len(groups), 8):
        chunk = b"".join(groups[start:start + 8])
        if len(chunk) < 8 * group_bytes:
            chunk += bytes(8 * group_bytes - len(chunk))
        raw = list(chunk)
        codes = oracle.unpack_codes(np.frombuffer(chunk, np.uint8), bits, 64)
        want = [entries[codes[2 * u]] | (entries[codes[2 * u + 1]] << 16) for u in range(32)]
        assert lookup_chunk(raw, bits, entries) == want, (bits, start)


def test_selector_nibbles_hold_the_codes_in_order():
    # 3 bits: nibble k of spread4(x) is code 3 - k of x (first code in the top bits)
    for x in range(4096):
        s = spread4(x, 3)
        assert [(s >> (4 * k)) & 15 for k in range(4)] == [(x >> (3 * k)) & 7 for k in range(4)]
        assert s < 1 << 16
    for x in range(256):
        s = spread4(x, 2)
        assert [(s >> (4 * k)) & 15 for k in range(4)] == [(x >> (2 * k)) & 3 for k in range(4)]
        assert s < 1 << 16
