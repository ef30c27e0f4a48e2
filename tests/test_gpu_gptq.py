"""GPU parity of llvq_spherical_gptq (one Spherical GPTQ pass, papernotes 关键设计 3) with the CPU
oracle's pass.

Both sides run the same fp64 operations in the same order (the order is part of the reading: the
norm as an fma chain, the retraction as a rounded product and difference, the block matrices by
back substitution, the update as an fma chain), and the search decides each direction on the
same fp32-rounded block, so the updated weights, norms and points must agree bit for bit.  A row
of zeros ties every direction: there only the weights and norms are compared.  Inputs: Gaussian
weights and a synthetic SPD Hessian from correlated inputs (X X^T / n plus damping); U is its
inverse's Cholesky factor from numpy, given to both sides.
"""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def codecs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import codebook_free_lattice_b200 as L
    return L.Codec(48), oracle.Codec(48)


def spd(rng, cols):
    X = rng.standard_normal((cols, 4 * cols)) * np.linspace(0.3, 2.0, cols)[:, None]
    X[1:] += 0.5 * X[:-1]
    H = X @ X.T / X.shape[1]
    return H + 0.05 * np.mean(np.diag(H)) * np.eye(cols)


def gpu_gptq(g, W, U, max_shell):
    rows, cols = W.shape
    Wd = torch.from_numpy(np.ascontiguousarray(W)).cuda()
    Ud = torch.from_numpy(np.ascontiguousarray(U)).cuda()
    P = torch.full((rows, cols // 24, 24), 99, dtype=torch.int8, device="cuda")
    N = torch.full((rows, cols // 24), float("nan"), dtype=torch.float64, device="cuda")
    g.spherical_gptq(Wd, Ud, P, N, max_shell)
    torch.cuda.synchronize()
    assert g.get_error() == 0
    return Wd.cpu().numpy(), P.cpu().numpy(), N.cpu().numpy()


CASES = [
    # rows, cols, max_shell
    (16, 24, 12),
    (24, 96, 8),
    (37, 240, 6),
    (12, 72, 13),
    (20, 144, 12),
]


@pytest.mark.parametrize("rows,cols,max_shell", CASES)
def test_gptq_matches_oracle_bit_for_bit(codecs, rows, cols, max_shell):
    g, o = codecs
    rng = np.random.default_rng(rows * 1000 + cols + max_shell)
    W = rng.standard_normal((rows, cols)) * rng.uniform(0.5, 2.0, (rows, 1))
    W[rows // 2] = 0.0                                   # a zero row: every direction ties
    U = np.linalg.cholesky(np.linalg.inv(spd(rng, cols))).T
    Wg, Pg, Ng = gpu_gptq(g, W, U, max_shell)
    Wo, Po, No = o.spherical_gptq(W, U, max_shell)
    assert np.array_equal(Ng, No), np.max(np.abs(Ng - No))
    assert np.array_equal(Wg, Wo), np.max(np.abs(Wg - Wo))
    keep = np.ones(rows, bool)
    keep[rows // 2] = False
    assert np.array_equal(Pg[keep], Po[keep])
    assert (Wg[rows // 2] == 0).all()


def test_gptq_arguments(codecs):
    import ctypes as C
    import codebook_free_lattice_b200 as L
    g, _ = codecs
    lib = L.lib()
    rows, cols = 8, 48
    need = lib.llvq_spherical_gptq_workspace(rows, cols)
    assert need >= cols * cols * 8 + rows * 36
    W = torch.zeros((rows, cols), dtype=torch.float64, device="cuda")
    U = torch.eye(cols, dtype=torch.float64, device="cuda")
    P = torch.zeros((rows, 2, 24), dtype=torch.int8, device="cuda")
    N = torch.zeros((rows, 2), dtype=torch.float64, device="cuda")
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    p = lambda t: C.c_void_p(t.data_ptr())
    call = lambda ms, r, c, nbytes: lib.llvq_spherical_gptq(g.handle, ms, r, c, p(W), p(U), p(P), p(N), p(ws),
                                                            nbytes, None)
    assert call(13, rows, cols, need) == L.LLVQ_OK
    assert call(13, rows, cols, need - 1) == L.LLVQ_ERR_ARG
    assert call(13, rows, 40, need) == L.LLVQ_ERR_ARG
    assert call(1, rows, cols, need) == L.LLVQ_ERR_ARG
    assert call(14, rows, cols, need) == L.LLVQ_ERR_ARG
    assert call(13, 0, cols, 0) == L.LLVQ_OK
    torch.cuda.synchronize()
    g72 = L.Codec(72)
    assert lib.llvq_spherical_gptq(g72.handle, 13, rows, cols, p(W), p(U), p(P), p(N), p(ws), need, None) == \
        L.LLVQ_ERR_UNSUPPORTED
