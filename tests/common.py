"""Shared helpers for the parity tests: synthetic layers (via the seeded generator) and the
error metric used for fp32-vs-fp64 comparisons."""
from __future__ import annotations

import numpy as np

from codebook_free_lattice_b200 import synth

# Tolerance of the fused products against the fp64 oracle: max relative error 2e-3, with
# rel_i = |y_i - ref_i| / max(|ref_i|, 1e-2 * rms(ref)) (the floor keeps outputs that cancel
# to nearly zero from dominating the relative error).
GEMV_RTOL = 2e-3


def max_rel_err(y: np.ndarray, ref: np.ndarray) -> float:
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    floor = 1e-2 * np.sqrt(np.mean(ref ** 2)) if ref.size else 0.0
    den = np.maximum(np.abs(ref), floor)
    den[den == 0] = 1.0
    return float(np.max(np.abs(y - ref) / den)) if ref.size else 0.0


class Layer:
    """A synthetic compressed layer: words [rows, nb(, 2)], fp16 gains, fp16 activations."""

    def __init__(self, index_bits, rows, K, batch, config_id, n_points, gain_mode,
                 index_limit=None, norms_fn=None, pitch=None, index_base=0):
        self.index_bits, self.rows, self.K, self.batch = index_bits, rows, K, batch
        self.nb = -(-K // 24)
        self.pitch = self.nb if pitch is None else pitch
        self.gain_mode = gain_mode
        limit = n_points if index_limit is None else index_limit
        lo, hi = synth.uniform_indices(synth.rng(config_id, 0), rows * self.pitch, limit - index_base, index_bits)
        if index_base:                          # uniform over [index_base, limit)
            blo = np.uint64(index_base & (2**64 - 1))
            lo2 = lo + blo
            hi = hi + np.uint64(index_base >> 64) + (lo2 < lo).astype(np.uint64)
            lo = lo2
        self.lo, self.hi = lo, hi
        codes = synth.gain_codes(synth.rng(config_id, 1), rows * self.pitch)
        self.codes = codes.reshape(rows, self.pitch)
        w = synth.pack_words(lo, hi, codes if gain_mode == 1 else None, index_bits)
        self.words = w.reshape((rows, self.pitch) + w.shape[1:])
        if gain_mode == 0:
            norms = norms_fn(lo, hi).reshape(rows, self.pitch)
            self.gains = synth.direct_gains(synth.rng(config_id, 1), norms)[:, :self.nb].copy()
        else:
            self.gains = synth.chi24_tables(synth.rng(config_id, 2), rows)
        self.x = synth.activations(synth.rng(config_id, 3), batch, K)
