"""Pins of the oracle's Spherical GPTQ pass (papernotes 关键设计 3: the shape-gain candidate is
rescaled to the original norm, w^ = (|w| / |w~|) w~, and the residual E = w - w^ is propagated to
the unquantized weights through U = chol(H^-1)^T).

Pinned against things that do not share the oracle's Cholesky arithmetic:
  * the block matrix G_B = U_BB^-1 U_B,rest equals the least-squares compensation from H itself,
    -H_{B,R} H_{R,R}^-1 (R = the later columns: the change D of the later columns that minimizes
    [-E, D] H [-E, D]^T is -E G_B), and the OBS form built from explicit inverses of the remaining
    Hessian;
  * one block alone is the retraction |w| v / |v| of the angular search, with the same norm;
  * two blocks equal a hand-run: search, retraction, the update through the H-form G, search;
  * the proxy loss tr(D H D^T) of the pass is below that of the same blockwise retraction
    without feedback, on every seeded instance (a sign or index error in the feedback raises it);
  * a diagonal Hessian couples no columns: the block matrices vanish and the pass is the
    blockwise retraction of the original weights.
"""
import numpy as np
import pytest

import oracle

ANG = oracle.ANGULAR


@pytest.fixture(scope="module")
def codec():
    return oracle.Codec(48)


def spd(rng, cols, cond=0.05):
    """A synthetic SPD Hessian like a calibration one: X X^T / n over correlated inputs, plus a
    small damping term."""
    X = rng.standard_normal((cols, 4 * cols)) * np.linspace(0.3, 2.0, cols)[:, None]
    X[1:] += 0.5 * X[:-1]                      # neighbouring inputs correlate
    H = X @ X.T / X.shape[1]
    return H + cond * np.mean(np.diag(H)) * np.eye(cols)


def chol_factor(H):
    return np.linalg.cholesky(np.linalg.inv(H)).T          # upper, H^-1 = U^T U


@pytest.mark.parametrize("cols,b", [(72, 0), (72, 1), (120, 2), (120, 3)])
def test_block_matrix_is_the_least_squares_compensation(cols, b):
    rng = np.random.default_rng(cols + b)
    H = spd(rng, cols)
    G = oracle.gptq_block_matrix(chol_factor(H), b)
    B = slice(24 * b, 24 * b + 24)
    R = slice(24 * b + 24, cols)
    ref = -H[B, R] @ np.linalg.inv(H[R, R])
    np.testing.assert_allclose(G[:, R], ref, rtol=0, atol=1e-9 * np.abs(ref).max())
    assert (G[:, : 24 * b + 24] == 0).all()
    # the OBS form: the inverse Hessian of the columns not yet quantized is inv(H[rem, rem])
    rem = slice(24 * b, cols)
    Hi = np.linalg.inv(H[rem, rem])
    obs = np.linalg.solve(Hi[:24, :24], Hi[:24, 24:])
    np.testing.assert_allclose(G[:, R], obs, rtol=0, atol=1e-9 * np.abs(obs).max())


def test_one_block_is_the_retraction(codec):
    rng = np.random.default_rng(3)
    W = rng.standard_normal((10, 24))
    U = chol_factor(spd(rng, 24))
    Wq, P, N = codec.spherical_gptq(W, U, 12)
    V, _ = codec.search(W.astype(np.float32), 12, ANG, 1.0)
    assert (P[:, 0] == V).all()
    n = np.linalg.norm(W, axis=1)
    np.testing.assert_allclose(N[:, 0], n, rtol=1e-15)
    ref = n[:, None] * V / np.linalg.norm(V.astype(np.float64), axis=1, keepdims=True)
    np.testing.assert_allclose(Wq, ref, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(np.linalg.norm(Wq, axis=1), n, rtol=1e-14)


def test_two_blocks_equal_a_hand_run(codec):
    rng = np.random.default_rng(4)
    cols = 48
    H = spd(rng, cols)
    W = rng.standard_normal((12, cols))
    Wq, P, N = codec.spherical_gptq(W, chol_factor(H), 8)
    # by hand: block 0
    V0, _ = codec.search(W[:, :24].astype(np.float32), 8, ANG, 1.0)
    n0 = np.linalg.norm(W[:, :24], axis=1)
    what0 = n0[:, None] * V0 / np.linalg.norm(V0.astype(np.float64), axis=1, keepdims=True)
    E = W[:, :24] - what0
    W1 = W[:, 24:] + E @ (H[:24, 24:] @ np.linalg.inv(H[24:, 24:]))      # -E G_B, H-form
    # block 1 on the updated weights
    V1, _ = codec.search(W1.astype(np.float32), 8, ANG, 1.0)
    n1 = np.linalg.norm(W1, axis=1)
    what1 = n1[:, None] * V1 / np.linalg.norm(V1.astype(np.float64), axis=1, keepdims=True)
    assert (P[:, 0] == V0).all() and (P[:, 1] == V1).all()
    np.testing.assert_allclose(Wq[:, :24], what0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Wq[:, 24:], what1, rtol=0, atol=1e-9)
    np.testing.assert_allclose(N, np.stack([n0, n1], 1), rtol=1e-12)


def retraction_only(codec, W, max_shell):
    out = np.empty_like(W)
    for b in range(W.shape[1] // 24):
        blk = W[:, 24 * b: 24 * b + 24]
        V, _ = codec.search(blk.astype(np.float32), max_shell, ANG, 1.0)
        n = np.linalg.norm(blk, axis=1)
        out[:, 24 * b: 24 * b + 24] = n[:, None] * V / np.linalg.norm(V.astype(np.float64), axis=1, keepdims=True)
    return out


@pytest.mark.parametrize("seed", range(4))
def test_feedback_lowers_the_proxy_loss(codec, seed):
    rng = np.random.default_rng(100 + seed)
    cols = 96
    H = spd(rng, cols)
    W = rng.standard_normal((16, cols))
    Wq, _, _ = codec.spherical_gptq(W, chol_factor(H), 6)
    Wr = retraction_only(codec, W, 6)
    loss = lambda D: float(np.trace(D @ H @ D.T))
    assert loss(Wq - W) < loss(Wr - W)


def test_diagonal_hessian_has_no_feedback(codec):
    """A diagonal Hessian couples no columns: every G_B is zero and the pass is exactly the
    blockwise retraction."""
    rng = np.random.default_rng(9)
    cols = 72
    H = np.diag(rng.uniform(0.5, 3.0, cols))
    U = chol_factor(H)
    for b in range(cols // 24):
        assert (oracle.gptq_block_matrix(U, b) == 0).all()
    W = rng.standard_normal((10, cols))
    Wq, P, N = codec.spherical_gptq(W, U, 8)
    # the later columns reach the search unchanged: the same points as on the original blocks
    for b in range(cols // 24):
        V, _ = codec.search(W[:, 24 * b: 24 * b + 24].astype(np.float32), 8, ANG, 1.0)
        assert (P[:, b] == V).all()
    np.testing.assert_allclose(N, np.linalg.norm(W.reshape(10, -1, 24), axis=2), rtol=1e-15)
    np.testing.assert_allclose(Wq, retraction_only(codec, W, 8), rtol=1e-15, atol=0)
