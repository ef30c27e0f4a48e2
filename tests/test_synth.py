"""The seeded input generator (shared by the tests, the bench and the smoke check) on the CPU:
indices stay inside the coded range and are uniform, the packed-word bit layout matches the
format (index in the low bits, gain code right above), and the gain tables and activations have
the documented shapes and ranges."""
import numpy as np
import pytest

from codebook_free_lattice_b200 import synth

N48 = 280974212784720
N72 = 4337307873470892771360
N96 = 74972166705387133681638419280


def as_int(lo, hi):
    return [int(h) << 64 | int(l) for l, h in zip(lo, hi)]


@pytest.mark.parametrize("n_points,bits", [(N48, 48), (N72, 72), (N96, 96), (1000, 48), (2**64 + 5, 72)])
def test_indices_in_range_and_deterministic(n_points, bits):
    lo, hi = synth.uniform_indices(synth.rng(3, 0), 20000, n_points, bits)
    vals = as_int(lo, hi)
    assert max(vals) < n_points and min(vals) >= 0
    lo2, hi2 = synth.uniform_indices(synth.rng(3, 0), 20000, n_points, bits)
    assert np.array_equal(lo, lo2) and np.array_equal(hi, hi2)
    lo3, _ = synth.uniform_indices(synth.rng(3, 1), 20000, n_points, bits)
    assert not np.array_equal(lo, lo3)                   # another stream gives other numbers


@pytest.mark.parametrize("n_points,bits", [(N48, 48), (N96, 96), (2**64 + 5, 72)])
def test_indices_are_uniform(n_points, bits):
    """Fraction below a threshold matches its share of the range (binomial, 6 sigma)."""
    n = 200_000
    lo, hi = synth.uniform_indices(synth.rng(4, 0), n, n_points, bits)
    vals = np.array([v / n_points for v in as_int(lo, hi)])
    for q in (0.01, 0.25, 0.5, 0.9):
        frac = float(np.mean(vals < q))
        assert abs(frac - q) < 6 * np.sqrt(q * (1 - q) / n)


def test_packed_word_layout():
    lo = np.array([0x123456789ABC, 5], np.uint64)
    codes = np.array([0xA5, 0xFF], np.uint8)
    w48 = synth.pack_words(lo, None, codes, 48)
    assert int(w48[0]) == 0xA5 << 48 | 0x123456789ABC and int(w48[1]) >> 56 == 0
    hi = np.array([0xAB, 0x12345678], np.uint64)
    w72 = synth.pack_words(lo, hi, codes, 72)
    assert int(w72[0, 0]) == 0x123456789ABC and int(w72[0, 1]) == 0xA5 << 8 | 0xAB
    w96 = synth.pack_words(lo, hi, codes, 96)
    assert int(w96[1, 1]) == 0xFF << 32 | 0x12345678
    assert synth.pack_words(lo, hi, None, 96)[1, 1] == 0x12345678


def test_gain_tables_codes_and_activations():
    codes = synth.gain_codes(synth.rng(5, 1), (300, 7))
    assert codes.dtype == np.uint8 and codes.shape == (300, 7)
    assert len(np.unique(codes)) > 200
    t = synth.chi24_tables(synth.rng(5, 2), 64).astype(np.float64)
    assert t.shape == (64, 256) and (t > 0).all() and (np.diff(t, axis=1) >= 0).all()
    # chi(24) quantiles scaled by sigma in [0.5, 2): the median entry lies near sigma sqrt(24)
    ratio = t[:, 128] / t[:, 128].min()
    assert ratio.max() < 4.0
    x = synth.activations(synth.rng(5, 3), 3, 1000)
    assert x.dtype == np.float16 and x.shape == (3, synth.k_pad(1000)) == (3, 1008)
    assert (x[:, 1000:] == 0).all() and np.abs(x[:, :1000]).mean() > 0.5
    assert synth.k_pad(4096) == 4104 and synth.k_pad(24) == 24


def test_direct_gains_follow_the_norms():
    norms = np.full((50, 20), 4 * np.sqrt(13.0))
    g = synth.direct_gains(synth.rng(6, 1), norms).astype(np.float64)
    assert g.shape == norms.shape and (g >= 0).all()
    # |z| sqrt(24) / norm with z ~ N(0, 1): mean sqrt(2/pi) sqrt(24) / norm
    assert abs(g.mean() - np.sqrt(2 / np.pi) * np.sqrt(24) / norms[0, 0]) < 0.05


def test_gaussian_blocks_seeded_unit_variance():
    a = synth.gaussian_blocks(synth.rng(61, 4), 50_000)
    b = synth.gaussian_blocks(synth.rng(61, 4), 50_000)
    assert a.dtype == np.float32 and a.shape == (50_000, 24) and np.array_equal(a, b)
    assert not np.array_equal(a[:100], synth.gaussian_blocks(synth.rng(60, 4), 100))
    assert abs(a.mean()) < 0.01 and abs(a.var() - 1.0) < 0.01            # N(0, 1), 1.2M samples
