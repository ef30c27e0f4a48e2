"""The bounded waits of the kernels, made to give up on purpose (no fault, no hang).

llvq_set_wait_polls sets how many polls a kernel's first wait on its table copy (and on each
round of its tensor-core products) makes before it gives up.  With 0 the first wait gives up at
once: the kernel must raise LLVQ_FLAG_WAIT_TIMEOUT, wait again (up to the default limit) for the
copy or the products still in flight, and return; the GPU must stay usable, which the same call
with the default limits then shows by matching the oracle.  Each kernel family that waits is
covered: the coset-sorted product and decode, the warp-binned product (long row ranges) and the
tensor-core product (batch >= 8).
"""
import numpy as np
import pytest

import oracle
from tests.common import GEMV_RTOL, Layer, max_rel_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def codecs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import codebook_free_lattice_b200 as L
    yield L.Codec(48), oracle.Codec(48)
    L.llvq_set_wait_polls()


def product(g, layer, batch):
    words = torch.from_numpy(np.ascontiguousarray(layer.words).view(np.int64)).cuda()
    gains = torch.from_numpy(layer.gains.view(np.int16)).cuda()
    X = torch.from_numpy(layer.x[:batch].view(np.int16)).cuda()
    Y = torch.zeros((batch, layer.rows), dtype=torch.float32, device="cuda")
    w = g.weight(words, gains, layer.rows, layer.K, layer.gain_mode, layer.pitch)
    if batch == 1:
        g.gemv(w, X, Y)
    else:
        g.gemm(w, X, Y, batch)
    torch.cuda.synchronize()
    return Y.cpu().numpy().astype(np.float64)


# (rows, K, batch, table polls, product polls): the coset-sorted product, the warp-binned product
# (>= 10000 blocks per SM), the tensor-core product's table wait and its per-round product wait
CASES = [(300, 24 * 40, 1, 0, None), (1480, 24 * 1024, 1, 0, None), (256, 24 * 24, 16, 0, None),
         (256, 24 * 24, 16, None, 0)]


@pytest.mark.parametrize("rows,K,batch,tpolls,mpolls", CASES)
def test_product_wait_gives_up_then_recovers(codecs, rows, K, batch, tpolls, mpolls):
    import codebook_free_lattice_b200 as L
    g, o = codecs
    layer = Layer(48, rows, K, batch, 990 + batch, o.n_points, 1)
    g.get_error()
    L.llvq_set_wait_polls(0xFFFFFFFF if tpolls is None else tpolls, 0xFFFFFFFF if mpolls is None else mpolls)
    try:
        product(g, layer, batch)
        assert g.get_error() & L.LLVQ_FLAG_WAIT_TIMEOUT
    finally:
        L.llvq_set_wait_polls()
    y = product(g, layer, batch)
    assert g.get_error() == 0
    rs = np.sort(np.random.default_rng(rows).choice(rows, 32, replace=False))
    ref = o.gemm(layer.words[rs], layer.nb, 1, layer.gains[rs], layer.x[:batch], batch)
    assert max_rel_err(y[:, rs], ref) < GEMV_RTOL


def test_decode_wait_gives_up_then_recovers(codecs):
    import codebook_free_lattice_b200 as L
    from codebook_free_lattice_b200 import synth
    g, o = codecs
    lo, _ = synth.uniform_indices(synth.rng(77, 0), 50_000, o.n_points, 48)
    w = torch.from_numpy(lo.view(np.int64)).cuda()
    out = torch.empty((lo.shape[0], 24), dtype=torch.int8, device="cuda")
    g.get_error()
    L.llvq_set_wait_polls(0, 0xFFFFFFFF)
    try:
        g.decode(w, out)
        torch.cuda.synchronize()
        assert g.get_error() & L.LLVQ_FLAG_WAIT_TIMEOUT
    finally:
        L.llvq_set_wait_polls()
    g.decode(w, out)
    torch.cuda.synchronize()
    assert g.get_error() == 0
    assert np.array_equal(out.cpu().numpy(), o.decode_batch(lo))
