"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module only draws random numbers. It holds none of the codec arithmetic: every value it returns
is either a random draw (with the torch CPU generator, so the draws are reproducible on any machine)
or a plain constant-fill. The random tables the two methods draw themselves are generated here with
the same generator calls the source pages use, so that both the CUDA path and the oracle receive them
as inputs:

* TQ3 sign flips: ``tq3_core.py``, ``_generate_sign_flips`` -- a CPU generator seeded with 42 draws
  ``randint(0, 2)`` over 128 positions; a drawn 1 means "+1", a drawn 0 means "-1".
* RPBH rotation: ``orbit_quant.py``, ``rpbh_params`` -- a CPU generator seeded with ``0x0EB17 + d``
  draws ``randperm(d)`` and then ``randint(0, 2)`` as int8, mapped to -1/+1 by ``2*b - 1``.

The workload recipes (shapes, distributions, seeds) are the benchmark configurations of this codec:
a 4096-vector TQ3 round trip, a bf16 KV cache of 8x8x4096x128 for K and for V, a 1M-record
long-context decode, and RPBH weights/activations shaped like an LLM MLP (11008 inputs) and a DiT
block (3072 inputs). Nothing here touches a GPU.
"""
from __future__ import annotations

import numpy as np
import torch

TQ3_SIGN_SEED = 42
RPBH_SEED_BASE = 0x0EB17


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


# ----------------------------------------------------------------------------------------------
# random tables the methods draw
# ----------------------------------------------------------------------------------------------
def tq3_sign_bits(seed: int = TQ3_SIGN_SEED) -> np.ndarray:
    """The 128 sign draws of ``_generate_sign_flips`` (uint8, 1 = keep sign, 0 = flip)."""
    bits = torch.randint(0, 2, (128,), generator=_gen(seed), dtype=torch.float32)
    return bits.numpy().astype(np.uint8)


def tq3_sign_mask_words(bits: np.ndarray) -> np.ndarray:
    """The same draws laid out as four little-endian 32-bit words, bit i of the 128-bit mask = draw i."""
    bits = np.asarray(bits, dtype=np.uint64).reshape(4, 32)
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (bits * weights).sum(axis=1).astype(np.uint32)


def rpbh_params(d: int) -> tuple[np.ndarray, np.ndarray]:
    """The RPBH permutation (int32) and Rademacher signs (int8, -1/+1) for input dimension d."""
    g = _gen(RPBH_SEED_BASE + d)
    perm = torch.randperm(d, generator=g)
    signs = torch.randint(0, 2, (d,), generator=g, dtype=torch.int8) * 2 - 1
    return perm.numpy().astype(np.int32), signs.numpy().astype(np.int8)


# ----------------------------------------------------------------------------------------------
# bf16 storage helpers (pure bit reinterpretation of torch's own bf16 cast)
# ----------------------------------------------------------------------------------------------
def to_bf16_bits(t: torch.Tensor) -> np.ndarray:
    """torch's round-to-nearest-even bf16 cast, returned as raw uint16 bit patterns."""
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------------------------------------
# workload recipes
# ----------------------------------------------------------------------------------------------
def tq3_roundtrip(n_gauss: int = 4064, n_const: int = 32, seed: int = 0) -> np.ndarray:
    """fp32 [n_gauss + n_const, 128]: i.i.d. N(0,1) rows followed by constant rows of value 1.0."""
    x = torch.randn(n_gauss, 128, generator=_gen(seed), dtype=torch.float32)
    c = torch.ones(n_const, 128, dtype=torch.float32)
    return torch.cat([x, c], 0).numpy()


def kv_cache(batch: int = 8, heads: int = 8, seq: int = 4096, head_dim: int = 128,
             seed: int = 1, n_outlier: int = 4, outlier_gain: float = 20.0,
             offset_std: float = 2.0) -> tuple[np.ndarray, np.ndarray]:
    """bf16 K and V caches [batch, heads, seq, head_dim] as uint16 bit patterns.

    Each of K and V is N(0,1) with ``n_outlier`` fixed channels (the first entries of one
    randperm(head_dim) draw, shared by K and V) multiplied by ``outlier_gain``, plus a per-token
    offset drawn from N(0, offset_std^2) added to every channel of that token.
    """
    g = _gen(seed)
    shape = (batch, heads, seq, head_dim)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    ch = torch.randperm(head_dim, generator=g)[:n_outlier]
    k_off = torch.randn((batch, heads, seq, 1), generator=g, dtype=torch.float32) * offset_std
    v_off = torch.randn((batch, heads, seq, 1), generator=g, dtype=torch.float32) * offset_std
    for t, off in ((k, k_off), (v, v_off)):
        t[..., ch] *= outlier_gain
        t += off
    return to_bf16_bits(k), to_bf16_bits(v)


def long_context_records(n_vec: int = 1 << 20, seed: int = 2) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """TQ3 records for a decode-only workload: packed uint8 [n_vec, 48], norms, scales (fp32).

    Indices uniform over 0..7 packed 3 bits each are exactly uniform random bytes, so the packed
    payload is drawn as bytes directly. Norms are |N(10, 2^2)|, scales U(0.1, 0.5).
    """
    g = _gen(seed)
    packed = torch.randint(0, 256, (n_vec, 48), generator=g, dtype=torch.uint8)
    norms = (torch.randn(n_vec, generator=g, dtype=torch.float32) * 2.0 + 10.0).abs()
    scales = torch.rand(n_vec, generator=g, dtype=torch.float32) * 0.4 + 0.1
    return packed.numpy(), norms.numpy(), scales.numpy()


def llm_weight(rows: int = 4096, d: int = 11008, seed: int = 3, frac_hot: float = 0.01,
               hot_gain: float = 8.0) -> np.ndarray:
    """bf16 W [rows, d] (uint16 bits): 0.02 * Student-t(3), with 1% of columns multiplied by 8.

    Student-t(3) is drawn explicitly as z / sqrt(chi2_3 / 3) with chi2_3 a sum of three squared
    normals, all from the seeded generator.
    """
    g = _gen(seed)
    z = torch.randn(rows, d, generator=g, dtype=torch.float32)
    chi = torch.zeros(rows, d, dtype=torch.float32)
    for _ in range(3):
        n = torch.randn(rows, d, generator=g, dtype=torch.float32)
        chi += n * n
    w = 0.02 * z / torch.sqrt(chi / 3.0)
    hot = torch.randperm(d, generator=g)[: int(frac_hot * d)]
    w[:, hot] *= hot_gain
    return to_bf16_bits(w)


def dit_weight(rows: int, d: int = 3072, seed: int = 4) -> np.ndarray:
    """bf16 W [rows, d] (uint16 bits): N(0, 0.02^2) entries times a per-row LogNormal(0, 0.5) scale."""
    g = _gen(seed)
    w = torch.randn(rows, d, generator=g, dtype=torch.float32) * 0.02
    row_scale = torch.exp(0.5 * torch.randn(rows, 1, generator=g, dtype=torch.float32))
    return to_bf16_bits(w * row_scale)


def activations(rows: int, d: int, seed: int) -> np.ndarray:
    """bf16 x [rows, d] (uint16 bits) ~ N(0, 1)."""
    return to_bf16_bits(torch.randn(rows, d, generator=_gen(seed), dtype=torch.float32))


def gaussian(shape, seed: int, dtype=torch.float32) -> np.ndarray:
    """Plain N(0,1) fp32 draws of any shape (small test cases)."""
    return torch.randn(tuple(shape), generator=_gen(seed), dtype=dtype).numpy()


def uniform_int(shape, high: int, seed: int) -> np.ndarray:
    """Integers uniform on [0, high) of any shape (uint8)."""
    return torch.randint(0, high, tuple(shape), generator=_gen(seed), dtype=torch.int64).numpy().astype(np.uint8)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32 values (bf16 is the top half of an fp32)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
