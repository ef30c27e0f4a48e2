"""GPU parity of llvq_search, the nearest-point search over the shell union Shell(2) u ... u
Shell(M) (papernotes 关键设计 1; gist.science Methodik 2), with the CPU oracle's search.

The CUDA kernel evaluates every class and codeword by a closed form in prefix sums of the sorted
|x_i|; the oracle builds each (class, codeword) candidate point explicitly and takes its dot
product.  Both are fp64, so the chosen points must be equal, except where two points are equally
good up to rounding (then both must be points of the union with the same criterion value).
Inputs: Gaussian rows (the workload of the pages' 2-bit Gaussian-source experiment) and
structured rows -- lattice points with small noise, basis vectors, rows with exact zeros and
repeated magnitudes, the zero row -- over unions 2..3 up to 2..13, both criteria, ragged sizes,
the empty call, non-finite rows, and the gain-level choice of the angular criterion.  The
full-size case (131,072 rows, the experiment's size, in the launch configuration the experiment
uses) checks every row for membership and sampled rows against the oracle.
"""
import os

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

ANG, EUC = oracle.ANGULAR, oracle.EUCLIDEAN
THREADS = os.cpu_count() or 1


@pytest.fixture(scope="module")
def codecs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import codebook_free_lattice_b200 as L
    return L.Codec(48), oracle.Codec(48)


def gpu_search(g, X, max_shell, mode, scale, levels=None):
    X = np.ascontiguousarray(X, np.float32).reshape(-1, 24)
    n = X.shape[0]
    Xd = torch.from_numpy(X).cuda()
    P = torch.full((max(n, 1), 24), 99, dtype=torch.int8, device="cuda")
    D = torch.full((max(n, 1),), float("nan"), dtype=torch.float64, device="cuda")
    lev = codes = None
    if levels is not None:
        lev = torch.tensor(levels, dtype=torch.float64, device="cuda")
        codes = torch.full((max(n, 1),), 255, dtype=torch.uint8, device="cuda")
    g.search(Xd, P, max_shell, mode, scale, dots=D, levels=lev, codes=codes, n=n)
    torch.cuda.synchronize()
    err = g.get_error()
    out = (P.cpu().numpy()[:n], D.cpu().numpy()[:n], err)
    return out + ((codes.cpu().numpy()[:n],) if codes is not None else ())


def norms(V):
    return (V.astype(np.int64) ** 2).sum(1)


_GOLAY = None


def in_union(V, max_shell):
    """Rows of V that are points of the scaled Leech lattice with shell in 2..max_shell (the
    textbook congruences: one parity; the 2-mod-4 (even) or 1-mod-4 (odd) positions form a
    codeword; sum 0 (even) or 4 (odd) mod 8)."""
    global _GOLAY
    if _GOLAY is None:
        _GOLAY = set(int(w) for w in oracle.golay_by_mask())
    V = V.astype(np.int64)
    par = V[:, :1] & 1
    ok = (V & 1 == par).all(1)
    res = np.where(par == 0, 2, 1)
    mask = ((V % 4 == res) * (1 << np.arange(24))).sum(1)
    ok &= np.array([int(m) in _GOLAY for m in mask])
    ok &= (V.sum(1) % 8) == np.where(par[:, 0] == 0, 0, 4)
    m = norms(V) // 16
    return ok & (norms(V) % 16 == 0) & (m >= 2) & (m <= max_shell)


def check(X, got, ref, mode, scale, max_shell):
    Vg, dg = got[0], got[1]
    Vo, do = ref
    X64 = X.astype(np.float64)
    assert in_union(Vg, max_shell).all()
    np.testing.assert_allclose(dg, (X64 * Vg).sum(1), rtol=0, atol=1e-12 * np.abs(X64).sum(1).max() * 16)
    fg = oracle.search_objective(mode, scale, (X64 * Vg).sum(1), norms(Vg))
    fo = oracle.search_objective(mode, scale, (X64 * Vo).sum(1), norms(Vo))
    tol = 1e-12 * np.maximum(1.0, np.abs(fo))
    assert (np.abs(fg - fo) <= tol).all(), np.max(np.abs(fg - fo))
    differ = ~(Vg == Vo).all(1)
    # where the points differ, the criterion ties within rounding (checked above); for inputs
    # drawn from a continuous distribution that happens at most on the deliberate tie rows
    return differ


def structured_rows(rng, ocodec, c):
    rows = []
    idx = rng.integers(0, ocodec.n_points, 6, dtype=np.uint64)
    P = ocodec.decode_batch(idx).astype(np.float64)
    rows += list(c * P + 0.05 * rng.standard_normal(P.shape))      # near lattice points
    rows += list(np.eye(24)[[0, 7, 23]])                            # basis vectors
    z = rng.standard_normal(24); z[rng.choice(24, 9, replace=False)] = 0.0
    rows.append(z)                                                  # exact zeros
    r = np.repeat(rng.standard_normal(6), 4) * rng.choice([-1, 1], 24)
    rows.append(r)                                                  # repeated magnitudes
    rows.append(np.round(rng.standard_normal(24) * 2) / 2)          # many ties
    return np.array(rows)


CASES = [
    # mode, scale, max_shell, gaussian rows
    (ANG, 1.0, 13, 77),
    (ANG, 1.0, 12, 40),
    (ANG, 1.0, 11, 40),
    (ANG, 1.0, 6, 40),
    (ANG, 1.0, 3, 40),
    (EUC, 0.30, 13, 77),
    (EUC, 0.20, 13, 40),
    (EUC, 0.45, 13, 40),
    (EUC, 0.60, 8, 40),
    (EUC, 0.50, 4, 40),
]


@pytest.mark.parametrize("mode,scale,max_shell,ngauss", CASES)
def test_search_matches_oracle(codecs, mode, scale, max_shell, ngauss):
    g, o = codecs
    rng = np.random.default_rng(1000 + 10 * max_shell + mode + int(scale * 100))
    X = np.concatenate([rng.standard_normal((ngauss, 24)),
                        structured_rows(rng, o, scale if mode == EUC else 1.0)]).astype(np.float32)
    got = gpu_search(g, X, max_shell, mode, scale)
    assert got[2] == 0
    ref = o.search(X, max_shell, mode, scale, threads=THREADS)
    differ = check(X, got, ref, mode, scale, max_shell)
    assert not differ[:ngauss].any()            # Gaussian rows: the same point


def test_zero_row_and_tie_rows(codecs):
    """The zero row ties every point (angular) or every shell-2 point (Euclidean): any point of
    the right set is correct."""
    g, o = codecs
    X = np.zeros((2, 24), np.float32)
    Va, da, err = gpu_search(g, X, 13, ANG, 1.0)
    assert err == 0 and in_union(Va, 13).all() and (da == 0).all()
    Ve, de, err = gpu_search(g, X, 13, EUC, 0.3)
    assert err == 0 and in_union(Ve, 13).all() and (norms(Ve) == 32).all()


def test_search_against_brute_force(codecs):
    """Shells 2..3 enumerated from the congruences, every point (16,969,680), against the GPU."""
    g, _ = codecs
    rng = np.random.default_rng(77)
    X = rng.standard_normal((24, 24)).astype(np.float32)
    for mode, scale in ((ANG, 1.0), (EUC, 0.35)):
        Vg, dg, err = gpu_search(g, X, 3, mode, scale)
        Vb, db, visited = oracle.search_brute(X, 3, mode, scale, threads=THREADS)
        assert err == 0 and visited == 16969680
        assert (Vg == Vb).all()
        np.testing.assert_allclose(dg, db, rtol=0, atol=1e-12)


def test_gain_codes(codecs):
    g, o = codecs
    rng = np.random.default_rng(88)
    X = rng.standard_normal((50, 24)).astype(np.float32)
    levels = [5.6, 3.9, 4.6, 4.6, 5.1]                   # unsorted, with a duplicate
    Vg, dg, err, codes = gpu_search(g, X, 12, ANG, 1.0, levels=levels)
    Vo, do = o.search(X, 12, ANG, 1.0, threads=THREADS)
    assert err == 0 and (Vg == Vo).all()
    gain = do / np.sqrt(norms(Vo))
    ref = np.argmin(np.abs(gain[:, None] - np.array(levels)[None, :]), axis=1)   # first of ties
    assert (codes == ref).all()


def test_ragged_empty_and_nonfinite(codecs):
    g, o = codecs
    rng = np.random.default_rng(99)
    X = rng.standard_normal((13, 24)).astype(np.float32)
    X[4, 7] = np.nan
    X[9, 0] = np.inf
    Vg, dg, err = gpu_search(g, X, 13, EUC, 0.3)
    assert err == 0x8                                   # LLVQ_FLAG_SEARCH_INPUT
    bad = np.zeros(13, bool); bad[[4, 9]] = True
    assert (Vg[bad] == 0).all() and np.isnan(dg[bad]).all()
    Vo, _ = o.search(X[~bad], 13, EUC, 0.3, threads=THREADS)
    assert (Vg[~bad] == Vo).all()
    V0, _, err = gpu_search(g, np.zeros((0, 24), np.float32), 13, ANG, 1.0)
    assert err == 0 and V0.shape == (0, 24)


def test_argument_checks(codecs):
    import codebook_free_lattice_b200 as L
    g, _ = codecs
    lib = L.lib()
    X = torch.zeros((4, 24), dtype=torch.float32, device="cuda")
    P = torch.zeros((4, 24), dtype=torch.int8, device="cuda")
    lv = torch.ones(4, dtype=torch.float64, device="cuda")
    cd = torch.zeros(4, dtype=torch.uint8, device="cuda")
    h = g.handle
    p = lambda t: None if t is None else t.data_ptr()
    call = lambda ms, mode, sc, levels=None, nl=0, codes=None, n=4: lib.llvq_search(
        h, ms, mode, sc, p(X), n, p(P), None, p(levels), nl, p(codes), None)
    assert call(13, ANG, 1.0) == L.LLVQ_OK
    assert call(1, ANG, 1.0) == L.LLVQ_ERR_ARG
    assert call(14, ANG, 1.0) == L.LLVQ_ERR_ARG
    assert call(13, 2, 1.0) == L.LLVQ_ERR_ARG
    assert call(13, EUC, 0.0) == L.LLVQ_ERR_ARG
    assert call(13, EUC, float("inf")) == L.LLVQ_ERR_ARG
    assert call(13, EUC, 0.3, lv, 4, cd) == L.LLVQ_ERR_ARG       # gain levels: angular only
    assert call(13, ANG, 1.0, lv, 0, cd) == L.LLVQ_ERR_ARG
    assert call(13, ANG, 1.0, lv, 257, cd) == L.LLVQ_ERR_ARG
    assert call(13, ANG, 1.0, lv, 4, None) == L.LLVQ_ERR_ARG
    assert call(13, ANG, 1.0, lv, 4, cd) == L.LLVQ_OK
    assert call(13, ANG, 1.0, n=-1) == L.LLVQ_ERR_ARG
    torch.cuda.synchronize()
    g72 = L.Codec(72)
    assert lib.llvq_search(g72.handle, 13, ANG, 1.0, p(X), 4, p(P), None, None, 0, None, None) == L.LLVQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("mode,scale,max_shell", [(ANG, 1.0, 12), (EUC, 0.30, 13)])
def test_full_size_gaussian(codecs, mode, scale, max_shell):
    """131,072 unit-variance Gaussian rows: every answer is a point of the union with a
    consistent dot; 48 sampled rows equal the oracle's."""
    g, o = codecs
    rng = np.random.default_rng(4242 + mode)
    X = rng.standard_normal((131072, 24)).astype(np.float32)
    Vg, dg, err = gpu_search(g, X, max_shell, mode, scale)
    assert err == 0
    assert in_union(Vg, max_shell).all()
    np.testing.assert_allclose(dg, (X.astype(np.float64) * Vg).sum(1), rtol=0, atol=1e-9)
    rows = np.sort(rng.choice(X.shape[0], 48, replace=False))
    Vo, do = o.search(X[rows], max_shell, mode, scale, threads=THREADS)
    assert (Vg[rows] == Vo).all()
