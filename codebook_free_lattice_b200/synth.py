"""Seeded synthetic inputs for LLVQ layers (shared by the tests, the bench and the smoke check).

This module only draws random numbers and lays bits out in the packed word format; it holds
none of the method's decode or product arithmetic.  Quantities that depend on the codec (the
number of coded points N_M, per-block vector norms) are passed in by the caller.

Recipe (seeds numpy.random.default_rng([20260313, config_id, stream])):
  stream 0  indices, uniform over [0, N_M) (rejection from N_M.bit_length() random bits)
  stream 1  8-bit gain codes (uniform; equiprobable quantile bins) or direct gains
  stream 2  per-row scale sigma_r ~ U[0.5, 2) of the chi(24) gain tables
  stream 3  activations x ~ N(0, 1) rounded to fp16, zero tail from K to K_pad
  stream 4  Gaussian-source blocks for the search: x ~ N(0, I_24) in fp32 (the pages' 2-bit
            Gaussian-source experiment: zero-mean, unit-variance i.i.d. coordinates)
Layer shapes follow Llama-2 linear layers; real weights are not available, so uniform indices
stand in for quantised weight blocks.
"""
from __future__ import annotations

import numpy as np

BASE_SEED = 20260313
BLOCK = 24                      # Leech lattice dimension: weights per block along K


def rng(config_id: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([BASE_SEED, int(config_id), int(stream)])


def k_pad(K: int) -> int:
    """K rounded up to whole 24-weight blocks."""
    return -(-K // BLOCK) * BLOCK


def uniform_indices(g: np.random.Generator, n: int, n_points: int, index_bits: int):
    """n indices uniform over [0, n_points) as (lo, hi) uint64 arrays (hi = 0 below 2^64).
    Draws n_points.bit_length() random bits per index and rejects values >= n_points."""
    assert 0 < n_points <= 2 ** index_bits
    lo = np.empty(n, np.uint64)
    hi = np.zeros(n, np.uint64)
    if n_points <= 2 ** 63:
        lo[:] = g.integers(0, n_points, size=n, dtype=np.uint64)
        return lo, hi
    hi_bits = max(n_points.bit_length() - 64, 0)
    np_lo, np_hi = n_points & (2**64 - 1), n_points >> 64
    filled = 0
    while filled < n:
        want = 2 * (n - filled) + 16
        a = g.integers(0, 2**63, size=want, dtype=np.uint64) << np.uint64(1)
        a |= g.integers(0, 2, size=want, dtype=np.uint64)
        b = g.integers(0, 2**hi_bits, size=want, dtype=np.uint64) if hi_bits else np.zeros(want, np.uint64)
        ok = (b < np.uint64(np_hi)) | ((b == np.uint64(np_hi)) & (a < np.uint64(np_lo)))
        a, b = a[ok], b[ok]
        take = min(n - filled, a.shape[0])
        lo[filled:filled + take] = a[:take]
        hi[filled:filled + take] = b[:take]
        filled += take
    return lo, hi


def pack_words(lo: np.ndarray, hi: np.ndarray, codes: np.ndarray | None, index_bits: int):
    """Packed words: index in the low index_bits bits, the 8-bit gain code right above it.
    48-bit indices give uint64 words [...]; 72/96-bit give little-endian uint64 pairs [..., 2]."""
    c = np.zeros(lo.shape, np.uint64) if codes is None else codes.astype(np.uint64)
    if index_bits == 48:
        return lo | (c << np.uint64(48))
    out = np.empty(lo.shape + (2,), np.uint64)
    out[..., 0] = lo
    out[..., 1] = hi | (c << np.uint64(index_bits - 64))
    return out


def gain_codes(g: np.random.Generator, shape) -> np.ndarray:
    return g.integers(0, 256, size=shape, dtype=np.uint8)


def chi24_tables(g: np.random.Generator, rows: int) -> np.ndarray:
    """Per-row 256-entry fp16 gain tables: sigma_r times the chi(24) quantiles at (j+0.5)/256
    (sorted ascending), sigma_r ~ U[0.5, 2) so that rows differ."""
    from scipy.stats import chi
    q = chi.ppf((np.arange(256) + 0.5) / 256.0, df=BLOCK)
    sigma = g.uniform(0.5, 2.0, size=rows)
    return (sigma[:, None] * q[None, :]).astype(np.float16)


def direct_gains(g: np.random.Generator, norms: np.ndarray) -> np.ndarray:
    """Per-block fp16 gains |z| * sqrt(24) / norm, z ~ N(0, 1); norm = |v| of each block."""
    z = np.abs(g.standard_normal(norms.shape))
    return (z * np.sqrt(BLOCK) / norms).astype(np.float16)


def activations(g: np.random.Generator, batch: int, K: int) -> np.ndarray:
    """fp16 activations [batch, K_pad], N(0, 1) on the first K columns, zero tail."""
    x = np.zeros((batch, k_pad(K)), np.float16)
    x[:, :K] = g.standard_normal((batch, K)).astype(np.float16)
    return x


def gaussian_blocks(g: np.random.Generator, n: int) -> np.ndarray:
    """n blocks of 24 i.i.d. zero-mean unit-variance Gaussian values, fp32 [n, 24]."""
    return g.standard_normal((n, BLOCK), dtype=np.float64).astype(np.float32)
