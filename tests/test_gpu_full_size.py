"""GPU parity of the fused products at the full sizes of the benchmark layers, on sampled rows.

Each case runs the whole layer through the C ABI with the launch configuration the bench uses
(the kernel is chosen by the library from the layer's size and batch) and compares a seeded
sample of rows, element by element, with the CPU oracle's fp64 product (max relative error 2e-3,
tests.common.max_rel_err).  Every output must be finite.  The shapes are the Llama-2 layers the
benchmark configurations name: 7B (q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008) and
70B (28672x8192, 8192x28672), K padded to a multiple of 24, at 2, 3 and 4 bits per weight with
per-row u8 gain tables and indices uniform over the whole budget.  The last cases run one
decoder layer of the 7B stack (seven products back to back on one stream) at each budget.
"""
import os

import numpy as np
import pytest

import oracle
from tests.common import GEMV_RTOL, Layer, max_rel_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

LLAMA7B_LAYER = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                 ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


_codecs = {}


def codecs(bits):
    """(GPU codec, oracle codec) for a budget, created once per module."""
    if bits not in _codecs:
        import codebook_free_lattice_b200 as L
        _codecs[bits] = (L.Codec(bits), oracle.Codec(bits))
    return _codecs[bits]


def launch(gcodec, layer, batch, stream=None):
    """The layer's product on the GPU; returns the device output (not synchronised)."""
    words = torch.from_numpy(np.ascontiguousarray(layer.words).view(np.int64)).cuda()
    gains = torch.from_numpy(layer.gains.view(np.int16)).cuda()
    X = torch.from_numpy(layer.x[:batch].view(np.int16)).cuda()
    Y = torch.full((batch, layer.rows), float("nan"), dtype=torch.float32, device="cuda")
    w = gcodec.weight(words, gains, layer.rows, layer.K, layer.gain_mode, layer.pitch)
    if batch == 1:
        gcodec.gemv(w, X, Y, stream=stream)
    else:
        gcodec.gemm(w, X, Y, batch, stream=stream)
    return Y, (words, gains, X)


def check_rows(ocodec, layer, y, nrows, seed, batch):
    rs = np.sort(np.random.default_rng(seed).choice(layer.rows, nrows, replace=False))
    ref = ocodec.gemm(layer.words[rs], layer.nb, layer.gain_mode, layer.gains[rs], layer.x[:batch], batch,
                      row_pitch_words=layer.pitch, threads=os.cpu_count() or 1)
    assert np.isfinite(y).all()
    err = max_rel_err(y[:, rs], ref)
    assert err < GEMV_RTOL, err


CASES = [
    # bits, rows, K, batch, sampled rows
    (48, 8192, 28672, 1, 128),
    (48, 8192, 28672, 16, 64),
    (48, 28672, 8192, 1, 128),
    (48, 28672, 8192, 2, 64),
    (48, 28672, 8192, 8, 64),
    (48, 11008, 4096, 1, 128),
    (48, 4096, 11008, 4, 64),
    (72, 4096, 4096, 1, 64),
    (72, 11008, 4096, 1, 64),
    (96, 4096, 4096, 1, 8),
    (96, 28672, 8192, 1, 6),
    (96, 8192, 28672, 1, 4),
    (96, 4096, 4096, 16, 4),
]


@pytest.mark.parametrize("bits,rows,K,batch,nrows", CASES)
def test_full_size_sampled_rows(dev, bits, rows, K, batch, nrows):
    g, o = codecs(bits)
    layer = Layer(bits, rows, K, batch, 700 + rows % 89 + batch, o.n_points, 1)
    Y, keep = launch(g, layer, batch)
    torch.cuda.synchronize()
    assert g.get_error() == 0
    check_rows(o, layer, Y.cpu().numpy().astype(np.float64), nrows, rows + K + batch, batch)


@pytest.mark.parametrize("bits,nrows,checked", [(48, 64, (0, 1, 2, 3, 4, 5, 6)), (72, 32, (0, 1, 2, 3, 4, 5, 6)),
                                                (96, 3, (0, 4, 6))])
def test_decoder_layer_stack(dev, bits, nrows, checked):
    """One decoder layer of the Llama-2-7B stack (q, k, v, o, gate, up, down) back to back on one
    stream, as the stack runs; the products are checked on sampled rows (at 4 bits, where the
    oracle builds every high shell's class list anew for each product, one product of each
    shape)."""
    g, o = codecs(bits)
    stream = torch.cuda.Stream()
    layers, outs, keep = [], [], []
    with torch.cuda.stream(stream):
        for i, (_, rows, K) in enumerate(LLAMA7B_LAYER):
            layer = Layer(bits, rows, K, 1, 800 + 10 * i + bits, o.n_points, 1)
            Y, k = launch(g, layer, 1, stream=stream)
            layers.append(layer)
            outs.append(Y)
            keep.append(k)
    stream.synchronize()
    assert g.get_error(stream) == 0
    for i, (layer, Y) in enumerate(zip(layers, outs)):
        y = Y.cpu().numpy().astype(np.float64)
        assert np.isfinite(y).all()
        if i in checked:
            check_rows(o, layer, y, nrows, 900 + i, 1)
