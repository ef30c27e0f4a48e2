"""Pins of the CPU oracle against facts other than itself (CPU only).

Each test states what it pins: the textbook Golay weight enumerator, the Leech theta series
(computed here from the closed form with Python integers), direct enumeration, brute force on
tiny inputs, lattice closure and integrality, and a dense numpy re-computation of the
fp64 product.  Page facts used: 4096 Golay codewords and the shell union m = 2..M
(papernotes.org notes, 关键设计 1-2), kissing number 196560 and about 0.75 bit per dimension
for the first shell (papernotes.org notes, 关键设计 1).
"""
import ctypes as C
import itertools
import math
import os

import numpy as np
import pytest

import oracle
from codebook_free_lattice_b200 import synth
from tests import theta

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def c48():
    return oracle.Codec(48)


@pytest.fixture(scope="module")
def c72():
    return oracle.Codec(72)


def popcount(a):
    a = a.astype(np.uint64)
    n = np.zeros(a.shape, np.int64)
    for b in range(24):
        n += ((a >> np.uint64(b)) & np.uint64(1)).astype(np.int64)
    return n


# ---------------------------------------------------------------- Golay code ----------------
def test_golay_weight_enumerator():
    """4096 distinct words with weights 1/759/2576/759/1 (textbook enumerator of G24)."""
    w = oracle.golay_by_mask()
    assert len(set(w.tolist())) == 4096
    counts = np.bincount(popcount(w), minlength=25)
    expect = np.zeros(25, np.int64)
    expect[[0, 8, 12, 16, 24]] = [1, 759, 2576, 759, 1]
    assert (counts == expect).all()


def test_golay_linear_self_orthogonal():
    """Closed under XOR (a linear code), pairwise even overlaps (self-orthogonal), min distance 8."""
    w = oracle.golay_by_mask().astype(np.uint64)
    s = set(w.tolist())
    rng = np.random.default_rng(0)
    a = w[rng.integers(0, 4096, 20000)]
    b = w[rng.integers(0, 4096, 20000)]
    assert all(int(x) in s for x in (a ^ b))
    overlap = popcount(w[:, None] & w[None, ::7])
    assert (overlap % 2 == 0).all()
    assert popcount(w[1:]).min() == 8


def test_golay_orders():
    """By-mask order is sorted; by-weight order groups weights with the stated bases."""
    bm = oracle.golay_by_mask()
    assert (np.diff(bm.astype(np.int64)) > 0).all()
    bw, base = oracle.golay_by_weight()
    assert sorted(bw.tolist()) == bm.tolist()
    wt = popcount(bw)
    assert list(base[[0, 8, 12, 16, 24, 25]]) == [0, 1, 760, 3336, 4095, 4096]
    for k, (lo, hi) in {0: (0, 1), 8: (1, 760), 12: (760, 3336), 16: (3336, 4095), 24: (4095, 4096)}.items():
        assert (wt[lo:hi] == k).all()
        assert (np.diff(bw[lo:hi].astype(np.int64)) > 0).all()


# ---------------------------------------------------------------- shells ---------------------
def test_theta_series_matches_dp_and_class_sums(c72):
    """Shell sizes three ways: theta closed form, coordinate DP, and sum of class sizes."""
    th = theta.leech_shell_sizes(60)
    dp = oracle.shell_counts_dp(60)
    assert th[2:61] == dp[2:61]
    assert th[2:5] == [196560, 16773120, 398034000]
    for m in range(2, c72.max_shell + 1):
        total = sum(c72.shell_class(m, j).size for j in range(c72.shell_nclasses(m)))
        assert total == th[m], m
        assert c72.shell_offset(m + 1) - c72.shell_offset(m) == th[m]


def test_no_roots_and_shell2_by_direct_search():
    """The lattice has no vectors of norm^2 2 (shell 1 empty) and 196560 minimal vectors, each
    a member with squared norm 32 in the sqrt(8) scaling."""
    assert oracle.shell_enumerate(1, store=False) == 0
    pts = oracle.shell_enumerate(2)
    assert pts.shape == (196560, 24)
    assert ((pts.astype(np.int64) ** 2).sum(1) == 32).all()
    assert len({tuple(p) for p in pts.tolist()}) == 196560
    for p in pts[::997]:
        assert oracle.in_leech(p)


def test_shell3_by_direct_search():
    assert oracle.shell_enumerate(3, store=False) == 16773120


@pytest.mark.slow
def test_shell4_by_direct_search():
    assert oracle.shell_enumerate(4, store=False) == 398034000


def test_shell2_class_split(c48):
    """Shell 2 = 97152 (2^8 0^16) + 1104 (4^2 0^22) + 98304 (odd 3 1^23)."""
    cl = [c48.shell_class(2, j) for j in range(c48.shell_nclasses(2))]
    assert [c.size for c in cl] == [97152, 1104, 98304]
    assert [(c.odd, c.vals, c.cnts) for c in cl] == [
        (False, [0, 2], [16, 8]), (False, [0, 4], [22, 2]), (True, [1, 3], [23, 1])]


def test_first_shell_rate():
    """log2(196560)/24 = 0.733 bit/dim, the pages' 'about 0.75 bit/dim' for the first shell."""
    assert abs(math.log2(196560) / 24 - 0.733) < 5e-4


@pytest.mark.parametrize("bits,M", [(48, 13), (72, 53), (96, 214)])
def test_budget_max_shell(bits, M):
    """M is the largest shell with N_2 + ... + N_M <= 2^bits (theta series)."""
    th = theta.leech_shell_sizes(M + 1)
    c = oracle.Codec(bits)
    assert c.max_shell == M
    n = sum(th[2:M + 1])
    assert c.n_points == n
    assert n <= 2 ** bits < n + th[M + 1]


def test_class_counts(c48, c72):
    assert sum(c48.shell_nclasses(m) for m in range(2, 14)) == 383
    assert sum(c72.shell_nclasses(m) for m in range(2, 54)) == 114976


def _class_formula_by_brute_force(c48, m):
    # a magnitude multiset is its count vector (how many coordinates have |x| = v, v = 0..15),
    # packed base 25 into one integer; the coset is the parity of the magnitudes
    mags = np.abs(oracle.shell_enumerate(m)).astype(np.int64)
    key = np.zeros(mags.shape[0], np.int64)
    for v in range(int(mags.max()), -1, -1):
        key = key * 25 + (mags == v).sum(axis=1)
    uniq, counts = np.unique(key, return_counts=True)
    found = dict(zip(uniq.tolist(), counts.tolist()))
    for j in range(c48.shell_nclasses(m)):
        cl = c48.shell_class(m, j)
        k = 0
        for v in range(int(mags.max()), -1, -1):
            k = k * 25 + dict(zip(cl.vals, cl.cnts)).get(v, 0)
        assert found.pop(k) == cl.size
        assert all(v % 2 == int(cl.odd) for v in cl.vals)
    assert not found


def test_class_formula_by_brute_force(c48):
    """Class size A * 2^B * P equals the number of enumerated shell-2 points with that
    magnitude multiset and coset (direct search, no class formula)."""
    _class_formula_by_brute_force(c48, 2)


@pytest.mark.slow
def test_class_formula_by_brute_force_shell3(c48):
    _class_formula_by_brute_force(c48, 3)


# ---------------------------------------------------------------- arrangements ---------------
@pytest.mark.parametrize("cnts", [[2, 1], [1, 1, 1, 1], [3, 2, 1], [2, 2, 2], [4, 1, 2], [1, 3]])
def test_arrangement_rank_is_lexicographic(cnts):
    """Unrank(k) is the k-th distinct permutation in lexicographic order (brute force)."""
    items = [g for g, n in enumerate(cnts) for _ in range(n)]
    perms = sorted(set(itertools.permutations(items)))
    for k, p in enumerate(perms):
        assert oracle.unrank_arrangement(cnts, k) == list(p)
        assert oracle.rank_arrangement(cnts, list(p)) == k
    with pytest.raises(ValueError):
        oracle.unrank_arrangement(cnts, len(perms))


# ---------------------------------------------------------------- the bijection --------------
def test_worked_examples(c48):
    with open(os.path.join(HERE, "golden", "worked_examples.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            head, vec = line.split(":")
            bits, idx = map(int, head.split())
            assert bits == 48
            assert c48.decode(idx) == list(map(int, vec.split()))


def test_exhaustive_bijection_shells_2_3(c48):
    """Every point of shells 2-3 (direct search) encodes into its shell's index range, each of
    the 16,969,680 indices is hit exactly once, and decode returns the point."""
    L = oracle.lib()
    L.ora_check_shells.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.POINTER(C.c_int64)]
    res = (C.c_int64 * 7)()
    rc = L.ora_check_shells(c48._h, 2, 3, os.cpu_count() or 1, res)
    assert list(res) == [16969680, 0, 0, 0, 0, 0, 0] and rc == 0


@pytest.mark.parametrize("bits", [48, 72, 96])
def test_decode_membership_and_roundtrip(bits):
    """Seeded uniform indices: decoded vectors satisfy the mod-2/4/8 congruences, have squared
    norm 16 m for their shell, and encode back to the index."""
    c = oracle.Codec(bits)
    n = {48: 4000, 72: 1500, 96: 2}[bits]
    lo, hi = synth.uniform_indices(synth.rng(99, bits), n, c.n_points, bits)
    shells = [m for m in range(2, c.max_shell + 2)]
    offs = [c.shell_offset(m) for m in shells]
    for a, b in zip(lo.tolist(), hi.tolist()):
        I = (int(b) << 64) | int(a)
        x = c.decode(I)
        assert oracle.in_leech(x)
        m = max(s for s, o in zip(shells, offs) if o <= I)
        assert sum(v * v for v in x) == 16 * m
        assert c.encode(x) == I


def test_lattice_closure_and_integrality(c48):
    """Sums/differences of decoded points are lattice points; inner products are multiples of 8
    (the sqrt(8)-scaled Leech lattice is even unimodular); off-lattice perturbations fail."""
    lo, _ = synth.uniform_indices(synth.rng(98, 0), 400, c48.n_points, 48)
    X = np.array([c48.decode(int(i)) for i in lo])
    for i in range(0, 400, 2):
        x, y = X[i], X[i + 1]
        assert oracle.in_leech(x + y) and oracle.in_leech(x - y)
        assert int(x @ y) % 8 == 0
        z = x.copy(); z[3] += 2
        assert not oracle.in_leech(z)           # breaks the mod-4 codeword pattern
        z = x.copy(); z[5] += 4
        assert not oracle.in_leech(z)           # breaks the mod-8 sum
        z = x.copy(); z[7] += 1
        assert not oracle.in_leech(z)           # breaks the common parity


# ---------------------------------------------------------------- the fp64 product -----------
def test_half_to_double_exact():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits[::37]])
    r = ref[::37]
    fin = np.isfinite(r)
    assert (got[fin] == r[fin]).all() and np.isnan(got[np.isnan(r)]).all()


def _layer(c, bits, rows, nb, seed, gain_mode):
    g = synth.rng(seed, 0)
    lo, hi = synth.uniform_indices(g, rows * nb, c.n_points, bits)
    codes = synth.gain_codes(synth.rng(seed, 1), rows * nb)
    words = synth.pack_words(lo, hi, codes if gain_mode == 1 else None, bits)
    words = words.reshape((rows, nb) + words.shape[1:])
    dec, shell, bad = c.decode_batch(lo, hi, with_shell=True)
    assert bad == 0
    if gain_mode == 0:
        norms = np.sqrt((dec.astype(np.float64) ** 2).sum(1))
        gains = synth.direct_gains(synth.rng(seed, 1), norms).reshape(rows, nb)
    else:
        gains = synth.chi24_tables(synth.rng(seed, 2), rows)
    return words, gains, dec.reshape(rows, nb, 24), codes.reshape(rows, nb)


@pytest.mark.parametrize("bits,gain_mode", [(48, 0), (48, 1), (72, 1)])
def test_gemm_matches_dense_numpy(bits, gain_mode):
    """The oracle product equals a dense fp64 matrix built from decoded blocks times gains,
    multiplied with numpy; the block norm comes from the decoded vector itself."""
    c = oracle.Codec(bits)
    rows, nb, batch = 37, 9, 3
    words, gains, dec, codes = _layer(c, bits, rows, nb, 7 + bits + gain_mode, gain_mode)
    x = synth.activations(synth.rng(5, 3), batch, nb * 24 - 5)
    y = c.gemm(words, nb, gain_mode, gains, x, batch)
    v = dec.astype(np.float64)
    if gain_mode == 0:
        scale = gains.astype(np.float64)
    else:
        t = gains.astype(np.float64)[np.arange(rows)[:, None], codes]
        scale = t / np.sqrt((v ** 2).sum(2))
    W = (scale[:, :, None] * v).reshape(rows, nb * 24)
    ref = x.astype(np.float64) @ W.T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_gemm_one_hot_is_decode(c48):
    """x = e_j gives y = gain * v at column j (ties the product to the decode)."""
    rows, nb = 11, 4
    words, gains, dec, _ = _layer(c48, 48, rows, nb, 21, 0)
    for j in (0, 29, 95):
        x = np.zeros((1, nb * 24), np.float16)
        x[0, j] = 1.0
        y = c48.gemm(words, nb, 0, gains, x, 1)[0]
        ref = gains[:, j // 24].astype(np.float64) * dec[:, j // 24, j % 24]
        assert (y == ref).all()


def test_gemm_batch_equals_repeated_gemv(c48):
    rows, nb, batch = 19, 6, 4
    words, gains, _, _ = _layer(c48, 48, rows, nb, 23, 1)
    x = synth.activations(synth.rng(6, 3), batch, nb * 24)
    y = c48.gemm(words, nb, 1, gains, x, batch)
    for b in range(batch):
        yb = c48.gemm(words, nb, 1, gains, x[b:b + 1], 1)[0]
        assert (yb == y[b]).all()
    ymt = c48.gemm(words, nb, 1, gains, x, batch, threads=3)
    assert (ymt == y).all()


def test_budgets_share_the_index_format():
    """Shell and class offsets do not depend on the budget: an index below N_13 decodes to the
    same vector at 48, 72 and 96 bits (the larger budgets only add shells above)."""
    from codebook_free_lattice_b200 import synth
    c48, c72, c96 = oracle.Codec(48), oracle.Codec(72), oracle.Codec(96)
    assert c72.shell_offset(14) == c96.shell_offset(14) == c48.n_points
    lo, _ = synth.uniform_indices(synth.rng(97, 0), 3000, c48.n_points, 48)
    lo = np.concatenate([lo, np.array([0, 196559, 196560, c48.n_points - 1], np.uint64)])
    v48 = c48.decode_batch(lo)
    assert np.array_equal(c72.decode_batch(lo, np.zeros_like(lo)), v48)
    assert np.array_equal(c96.decode_batch(lo, np.zeros_like(lo)), v48)
