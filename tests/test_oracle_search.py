"""Pins of the oracle's nearest-point search over the shell union Shell(2) u ... u Shell(M).

The search (papernotes 关键设计 1, 多壳层球面与角度搜索; gist.science Methodik 2: angular
criterion for the shape of a shape-gain split, Euclidean criterion for spherical clipping) takes
the best point of every class and Golay codeword by the rearrangement rules.  It is pinned here by
things that do not share those rules:
  * brute force over every point of shells 2..3 and 2..4, enumerated from the lattice
    congruences alone;
  * exact answers: a lattice point (times the scale) plus noise inside the packing radius is its
    own nearest point; the angular answer at a point's direction is that direction; the basis
    vector e_i has the shell-4 point 8 e_i (cosine 1) as its angular answer;
  * covariance under automorphisms of the lattice (the cyclic shift of coordinates 0..22, which
    maps the cyclic Golay code onto itself, a sign change on the positions of a weight-8
    codeword, and negation): searching the transformed input gives the transformed answer;
  * local optimality on the full 48-bit union (M = 13), where brute force is out of reach: no
    neighbour v + u, u one of the 196,560 minimal vectors, inside the union does better.
"""
import numpy as np
import pytest

import oracle

ANG, EUC = oracle.ANGULAR, oracle.EUCLIDEAN


@pytest.fixture(scope="module")
def codec():
    return oracle.Codec(48)


@pytest.fixture(scope="module")
def shell2():
    pts = oracle.shell_enumerate(2).astype(np.int64)
    assert pts.shape == (196560, 24)
    return pts


def norms(V):
    return (V.astype(np.int64) ** 2).sum(1)


def objective(mode, scale, X, V):
    d = (X.astype(np.float64) * V.astype(np.float64)).sum(1)
    return oracle.search_objective(mode, scale, d, norms(V))


def check_same_or_tied(codec_res, brute_res, X, mode, scale):
    """Both answers are lattice points of the union with the same objective; they are equal
    unless the objective ties (never for these continuous inputs, so equality is required)."""
    (V, d), (Vb, db) = codec_res, brute_res
    for v in V:
        assert oracle.in_leech(v.astype(np.int32))
    f, fb = objective(mode, scale, X, V), objective(mode, scale, X, Vb)
    np.testing.assert_allclose(d, (X.astype(np.float64) * V).sum(1), rtol=0, atol=1e-12)
    assert np.allclose(f, fb, rtol=1e-13, atol=1e-13)
    assert (V == Vb).all()


def mixed_targets(rng, n, codec, noise):
    """Half Gaussian rows, half lattice points of shells 2-3 with Gaussian noise."""
    g = rng.standard_normal((n - n // 2, 24))
    idx = rng.integers(0, codec.shell_offset(4), n // 2).astype(np.uint64)
    pts = codec.decode_batch(idx).astype(np.float64)
    return np.concatenate([g, pts * 0.25 + noise * rng.standard_normal(pts.shape)]).astype(np.float32)


@pytest.mark.parametrize("mode,scale", [(ANG, 1.0), (EUC, 0.25), (EUC, 0.4), (EUC, 0.8)])
def test_matches_brute_force_shells_2_3(codec, mode, scale):
    rng = np.random.default_rng(11 + int(scale * 100))
    X = mixed_targets(rng, 24, codec, 0.6)
    X[:4] *= np.float32(2.0)                 # far targets: the union clips them
    res = codec.search(X, 3, mode, scale, threads=8)
    Vb, db, visited = oracle.search_brute(X, 3, mode, scale, threads=8)
    assert visited == 196560 + 16773120
    check_same_or_tied(res, (Vb, db), X, mode, scale)
    shells = set(norms(res[0]) // 16)
    assert shells <= {2, 3} and (shells == {2, 3} or (mode, scale) != (EUC, 0.8))


def test_matches_brute_force_shells_2_4(codec):
    """Every point of shells 2..4 (415,003,680 points) for both criteria; the Euclidean targets
    have radii spread so that each of the three shells wins somewhere."""
    rng = np.random.default_rng(5)
    X = mixed_targets(rng, 10, codec, 0.5)
    res = codec.search(X, 4, ANG, 1.0, threads=8)
    Vb, db, visited = oracle.search_brute(X, 4, ANG, 1.0, threads=8)
    assert visited == 415003680
    check_same_or_tied(res, (Vb, db), X, ANG, 1.0)
    u = rng.standard_normal((10, 24))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    X2 = (u * np.linspace(5.2, 9.5, 10)[:, None] * 0.5).astype(np.float32)
    res2 = codec.search(X2, 4, EUC, 0.5, threads=8)
    Vb2, db2, _ = oracle.search_brute(X2, 4, EUC, 0.5, threads=8)
    check_same_or_tied(res2, (Vb2, db2), X2, EUC, 0.5)
    assert set(norms(res2[0]) // 16) == {2, 3, 4}


def test_lattice_points_are_their_own_answers(codec):
    rng = np.random.default_rng(21)
    idx = rng.integers(0, codec.n_points, 48, dtype=np.uint64)
    idx[:8] = rng.integers(0, codec.shell_offset(3), 8).astype(np.uint64)
    P = codec.decode_batch(idx).astype(np.float64)
    c = 0.3
    noise = rng.standard_normal(P.shape)
    noise *= (0.9 * c * np.sqrt(32) / 2 / np.linalg.norm(noise, axis=1, keepdims=True))
    X = (c * P + noise).astype(np.float32)                # inside the packing radius
    V, _ = codec.search(X, 13, EUC, c, threads=8)
    assert (V == P).all()
    X2 = (P + 1e-4 * rng.standard_normal(P.shape)).astype(np.float32)
    V2, _ = codec.search(X2, 13, ANG, 1.0, threads=8)
    # the angular answer has the same direction (it may be a multiple, such as 2v, in the union)
    dots = (V2.astype(np.int64) * P.astype(np.int64)).sum(1)
    assert (dots > 0).all() and (dots ** 2 == norms(V2) * norms(P.astype(np.int64))).all()


def test_basis_vectors(codec):
    X = np.eye(24, dtype=np.float32)
    V, d = codec.search(X, 13, ANG, 1.0, threads=8)
    assert (V == 8 * np.eye(24, dtype=np.int8)).all() and (d == 8).all()
    # below shell 4 no point has the direction of e_i.  Largest |x_i| / |x| there: shell 2
    # allows |x_i| <= 4 (4 / sqrt(32)); in shell 3 a 6 would need seven more 2-mod-4
    # coordinates (norm 64), while (5, 1, ..., 1) is a point (odd coset, 1-mod-4 set = all 24
    # coordinates, sum 28 = 4 mod 8): cosine 5 / sqrt(48).  Many sign patterns tie.
    V3, d3 = codec.search(X, 3, ANG, 1.0, threads=8)
    assert np.allclose(d3 / np.sqrt(norms(V3)), 5 / np.sqrt(48), rtol=0, atol=1e-15)
    assert all(oracle.in_leech(v.astype(np.int32)) for v in V3)
    V4, _ = codec.search(np.float32(8.0) * X, 13, EUC, 1.0, threads=8)
    assert (V4 == 8 * np.eye(24, dtype=np.int8)).all()


def _cyclic(x):
    """Coordinates 0..22 shifted by one (coordinate 23, the parity bit, stays)."""
    y = x.copy()
    y[..., 1:23] = x[..., 0:22]
    y[..., 0] = x[..., 22]
    return y


@pytest.mark.parametrize("mode,scale", [(ANG, 1.0), (EUC, 0.3)])
def test_automorphism_covariance(codec, mode, scale):
    rng = np.random.default_rng(31 + mode)
    X = rng.standard_normal((12, 24)).astype(np.float32)
    V, _ = codec.search(X, 13, mode, scale, threads=8)
    g = oracle.golay_by_mask()
    # the cyclic shift maps the code onto itself (the code's generator is a cyclic code on 0..22)
    gs = set(int(w) for w in g)
    sh = [sum(((int(w) >> i) & 1) << j for i, j in zip(range(24), list(range(1, 23)) + [0, 23])) for w in g]
    assert set(sh) == gs
    Vc, _ = codec.search(_cyclic(X), 13, mode, scale, threads=8)
    assert (Vc == _cyclic(V)).all()
    octad = next(int(w) for w in g if bin(int(w)).count("1") == 8)
    sgn = np.array([-1 if octad >> i & 1 else 1 for i in range(24)], np.float32)
    Vs, _ = codec.search(X * sgn, 13, mode, scale, threads=8)
    assert (Vs == V * sgn.astype(np.int8)).all()
    Vn, _ = codec.search(-X, 13, mode, scale, threads=8)
    assert (Vn == -V).all()


@pytest.mark.parametrize("mode,scale", [(ANG, 1.0), (EUC, 0.3), (EUC, 0.2)])
def test_local_optimality_full_union(codec, shell2, mode, scale):
    rng = np.random.default_rng(41 + int(10 * scale))
    X = rng.standard_normal((12, 24)).astype(np.float32)
    V, d = codec.search(X, 13, mode, scale, threads=8)
    f = objective(mode, scale, X, V)
    for x, v, fv in zip(X.astype(np.float64), V.astype(np.int64), f):
        W = v[None, :] + shell2
        nW = (W ** 2).sum(1)
        inside = (nW >= 32) & (nW <= 16 * 13)
        fw = oracle.search_objective(mode, scale, W[inside] @ x, nW[inside])
        assert fw.max() <= fv + 1e-12


def _assignment_best(y, mags_in, mags_out, in_set, signs_free_parity=None):
    """Largest sum_i y_i v_i by an exact assignment solver (scipy), for magnitudes placed on a
    set and its complement.  Odd classes pass the sign of each (position, magnitude) pair via
    signs_free_parity=None and in_set = the 1-mod-4 set T: v_i = +a when (a = 1 mod 4) equals
    (i in T).  Even classes pass signs_free_parity = (parity of the negative signs wanted on S);
    signs follow y, with one sign on S turned when the parity is wrong (more turns cost more)."""
    from scipy.optimize import linear_sum_assignment
    y = np.asarray(y, np.float64)
    if signs_free_parity is None:                       # odd: one 24 x 24 assignment
        a = np.asarray(mags_in, np.float64)
        sgn = np.where((np.asarray(mags_in)[None, :] % 4 == 1) == in_set[:, None], 1.0, -1.0)
        W = y[:, None] * sgn * a[None, :]
        r, c = linear_sum_assignment(W, maximize=True)
        return W[r, c].sum()
    S = np.flatnonzero(in_set)
    C_ = np.flatnonzero(~in_set)
    total = 0.0
    if C_.size:
        W = np.abs(y[C_])[:, None] * np.asarray(mags_out, np.float64)[None, :]
        r, c = linear_sum_assignment(W, maximize=True)
        total += W[r, c].sum()
    if S.size:
        WS = np.abs(y[S])[:, None] * np.asarray(mags_in, np.float64)[None, :]
        neg = int((y[S] < 0).sum())
        if neg % 2 == signs_free_parity:
            r, c = linear_sum_assignment(WS, maximize=True)
            total += WS[r, c].sum()
        else:
            best = -np.inf
            for t in range(S.size):                      # the turned sign on position S[t]
                W2 = WS.copy()
                W2[t] *= -1
                r, c = linear_sum_assignment(W2, maximize=True)
                best = max(best, W2[r, c].sum())
            total += best
    return total


def test_class_rules_against_assignment_solver(codec):
    """Every class of the 48-bit union, with random codewords and the extreme ones (the
    all-ones word and, for odd classes, the empty word, which put every position in one set
    and so force the largest surpluses): the rearrangement rules give the exact optimum of the
    assignment problem, computed by an independent solver."""
    rng = np.random.default_rng(51)
    g = np.asarray(oracle.golay_by_mask(), np.int64)
    wt = np.array([bin(int(w)).count("1") for w in g])
    ntested = 0
    for m in range(2, codec.max_shell + 1):
        for j in range(codec.shell_nclasses(m)):
            cl = codec.shell_class(m, j)
            mags = np.repeat(cl.vals, cl.cnts)
            if cl.odd:
                words = [0, 0xFFFFFF] + list(rng.choice(g, 2))
            else:
                pool = g[wt == cl.k]
                words = list(rng.choice(pool, min(2, pool.size)))
            for w in words:
                for trial in range(2):
                    y = rng.standard_normal(24)
                    if trial == 1:
                        y = np.abs(y) if rng.random() < 0.5 else -np.abs(y)
                    v, d = codec.class_best(m, j, int(w), y)
                    assert oracle.in_leech(v) and (v.astype(np.int64) ** 2).sum() == 16 * m
                    assert sorted(np.abs(v)) == sorted(mags)
                    in_set = np.array([(int(w) >> i) & 1 for i in range(24)], bool)
                    if cl.odd:
                        assert all(((v[i] % 4) == 1) == in_set[i] for i in range(24))
                        ref = _assignment_best(y, mags, None, in_set)
                    else:
                        assert (((np.abs(v) % 4) == 2) == in_set).all()
                        on = mags[mags % 4 == 2]
                        off = mags[mags % 4 == 0]
                        # sum = 0 mod 8 fixes the parity of the negative signs on S: a
                        # 2-mod-4 value changes the sum by 4 mod 8 when turned, a 0-mod-4 one by
                        # 0, so the parity is that of (sum of the magnitudes) / 4
                        par = (int(mags.sum()) // 4) % 2 if on.size else 0
                        ref = _assignment_best(y, on, off, in_set, par)
                    assert abs(d - ref) <= 1e-12 * max(1.0, abs(ref)), (m, j, int(w), d, ref)
                    ntested += 1
    assert ntested > 1500


def test_degenerate_targets_against_brute_force(codec):
    """Targets with exact zeros, repeated magnitudes, integer and half-integer entries and a wide
    range of scales (many equally good points): the search's criterion value equals brute force's
    over shell 2 and over shells 2..3 for both criteria, and its answer is a point of the union.
    Only the value is unique here, so the points themselves are not compared."""
    rng = np.random.default_rng(61)
    rows = []
    for t in range(40):
        kind = t % 5
        if kind == 0:
            x = rng.integers(-3, 4, 24).astype(np.float64)              # integers, many zeros and ties
        elif kind == 1:
            x = np.round(rng.standard_normal(24) * 2) / 2                # half-integers
        elif kind == 2:
            x = np.repeat(rng.standard_normal(3), 8)                     # three magnitudes, 8 times each
            x *= rng.choice([-1, 1], 24)
        elif kind == 3:
            x = rng.standard_normal(24)
            x[rng.choice(24, 20, replace=False)] = 0.0                   # sparse
        else:
            x = rng.standard_normal(24) * 10.0 ** rng.uniform(-3, 3)     # tiny to large scale
        rows.append(x)
    X = np.array(rows, np.float32)
    for m_max in (2, 3):
        for mode, scale in ((ANG, 1.0), (EUC, 0.35)):
            V, d = codec.search(X, m_max, mode, scale, threads=8)
            Vb, db, _ = oracle.search_brute(X, m_max, mode, scale, threads=8)
            n = norms(V)
            assert ((n >= 32) & (n <= 16 * m_max)).all()
            for v in V:
                assert oracle.in_leech(v.astype(np.int32))
            f, fb = objective(mode, scale, X, V), objective(mode, scale, X, Vb)
            np.testing.assert_allclose(f, fb, rtol=1e-12, atol=1e-12)
