"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Decoded lattice vectors must match bit for bit; fused products must be within max relative
error 2e-3 of the oracle's fp64 result (tests.common.max_rel_err).  Inputs come from the
seeded generator, sized so the oracle finishes in seconds while spanning many CTAs and ragged
tails; the full-size layers are checked on sampled rows.
"""
import os

import numpy as np
import pytest

import oracle
from codebook_free_lattice_b200 import synth
from tests.common import GEMV_RTOL, Layer, max_rel_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from codebook_free_lattice_b200 import build
    build.build()
    return torch.device("cuda:0")


@pytest.fixture(scope="module")
def gcodec(dev):
    import codebook_free_lattice_b200 as L
    return L.Codec(48)


@pytest.fixture(scope="module")
def ocodec():
    return oracle.Codec(48)


@pytest.fixture(scope="module")
def gcodec72(dev):
    import codebook_free_lattice_b200 as L
    return L.Codec(72)


@pytest.fixture(scope="module")
def ocodec72():
    return oracle.Codec(72)


def gpu_decode(gcodec, words_np):
    w = torch.from_numpy(np.ascontiguousarray(words_np).view(np.int64)).cuda()
    out = torch.empty((words_np.shape[0], 24), dtype=torch.int8, device="cuda")
    gcodec.decode(w, out, n=words_np.shape[0])
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_codec_info_matches_oracle(gcodec, ocodec):
    assert gcodec.max_shell == ocodec.max_shell == 13
    assert gcodec.n_points == ocodec.n_points == 280974212784720
    assert gcodec.n_classes == 383


def test_decode_shell2_all_and_shells_2_4_uniform(gcodec, ocodec):
    """All 196560 shell-2 indices, then 65536 seeded uniform indices over shells 2..4."""
    idx = np.arange(196560, dtype=np.uint64)
    lo, _ = synth.uniform_indices(synth.rng(1, 0), 65536, 415003680, 48)
    idx = np.concatenate([idx, lo])
    got = gpu_decode(gcodec, idx)
    ref = ocodec.decode_batch(idx)
    assert np.array_equal(got, ref)
    assert gcodec.get_error() == 0


def test_decode_uniform_full_budget(gcodec, ocodec):
    lo, _ = synth.uniform_indices(synth.rng(2, 0), 300_000, ocodec.n_points, 48)
    codes = synth.gain_codes(synth.rng(2, 1), lo.shape[0])
    words = synth.pack_words(lo, None, codes, 48)          # gain bits must be ignored
    got = gpu_decode(gcodec, words)
    assert np.array_equal(got, ocodec.decode_batch(lo))


def test_decode_class_boundaries(gcodec, ocodec):
    """First and last index of every class (and the last coded index)."""
    idx = []
    for c in ocodec.classes():
        idx += [c.offset, c.offset + c.size - 1, c.offset + c.size // 2]
    idx = np.array(idx, dtype=np.uint64)
    assert np.array_equal(gpu_decode(gcodec, idx), ocodec.decode_batch(idx))


@pytest.mark.parametrize("n", [0, 1, 31, 33, 513, 4097])
def test_decode_ragged_sizes(gcodec, ocodec, n):
    lo, _ = synth.uniform_indices(synth.rng(3, n), max(n, 1), ocodec.n_points, 48)
    lo = lo[:n]
    if n == 0:
        out = torch.full((4, 24), 7, dtype=torch.int8, device="cuda")
        gcodec.decode(torch.zeros(1, dtype=torch.int64, device="cuda"), out, n=0)
        torch.cuda.synchronize()
        assert (out.cpu() == 7).all()
        return
    assert np.array_equal(gpu_decode(gcodec, lo), ocodec.decode_batch(lo))


def test_decode_out_of_range_sets_flag(gcodec, ocodec):
    N = ocodec.n_points
    idx = np.array([0, N - 1, N, N + 12345, 2**48 - 1, 5], dtype=np.uint64)
    got = gpu_decode(gcodec, idx)
    assert gcodec.get_error() == 1
    ref = ocodec.decode_batch(idx)             # the oracle writes zero rows for bad indices
    assert np.array_equal(got, ref)
    assert (got[2:5] == 0).all()
    assert gcodec.get_error() == 0             # cleared by the previous read


# ------------------------------------------------------------------ encode (48-bit) --------

def gpu_encode(gcodec, vecs):
    v = torch.from_numpy(np.ascontiguousarray(vecs, np.int8)).cuda()
    w = torch.full((vecs.shape[0],), -1, dtype=torch.int64, device="cuda")
    gcodec.encode(v, w)
    torch.cuda.synchronize()
    return w.cpu().numpy().view(np.uint64)


def test_encode_roundtrip_uniform(gcodec, ocodec):
    """300,000 seeded uniform indices, decoded by the oracle, encode back to themselves."""
    lo, _ = synth.uniform_indices(synth.rng(70, 0), 300_000, ocodec.n_points, 48)
    vecs = ocodec.decode_batch(lo)
    assert np.array_equal(gpu_encode(gcodec, vecs), lo)
    assert gcodec.get_error() == 0


def test_encode_class_boundaries_and_oracle_encode(gcodec, ocodec):
    """First, middle and last index of every class; each result also equals the oracle's encode."""
    idx = []
    for c in ocodec.classes():
        idx += [c.offset, c.offset + c.size // 2, c.offset + c.size - 1]
    idx = np.array(idx, dtype=np.uint64)
    vecs = ocodec.decode_batch(idx)
    got = gpu_encode(gcodec, vecs)
    assert np.array_equal(got, idx)
    for t in range(0, len(idx), 7):
        assert int(got[t]) == ocodec.encode(vecs[t].astype(np.int32))


def test_encode_not_coded(gcodec, ocodec):
    """Vectors outside the coded set get 2^48 - 1 and raise the flag; the others in the same call
    still encode exactly."""
    lo, _ = synth.uniform_indices(synth.rng(71, 0), 64, ocodec.n_points, 48)
    good = ocodec.decode_batch(lo)
    bad = [np.zeros(24, np.int8)]                                   # zero vector
    v = good[0].copy(); v[3] += 2; bad.append(v)                    # breaks the congruences
    v = good[1].copy(); v[0] = -v[0] if v[0] else 4; bad.append(v)  # flips one sign / off-lattice
    small = ocodec.decode_batch(np.array([98256], np.uint64))[0]    # shell 2, odd
    bad.append((small * 4).astype(np.int8))                         # shell 32 > 13
    v = good[2].copy(); v[5] ^= 1; bad.append(v)                    # mixed parity
    bad = np.stack(bad)
    oracle_bad = []
    for b_ in bad:
        try:
            ocodec.encode(b_.astype(np.int32))
            oracle_bad.append(False)
        except ValueError:
            oracle_bad.append(True)
    vecs = np.concatenate([good[:10], bad, good[10:]])
    got = gpu_encode(gcodec, vecs)
    assert gcodec.get_error() == 4
    nb = len(bad)
    assert np.array_equal(got[:10], lo[:10]) and np.array_equal(got[10 + nb:], lo[10:])
    for t in range(nb):
        if oracle_bad[t]:
            assert int(got[10 + t]) == 2**48 - 1
        else:                                                       # a coded point after all
            assert int(got[10 + t]) == ocodec.encode(bad[t].astype(np.int32))
    assert all(oracle_bad[t] for t in (0, 1, 3, 4))


@pytest.mark.parametrize("n", [0, 1, 33, 513, 4097])
def test_encode_ragged_sizes(gcodec, ocodec, n):
    lo, _ = synth.uniform_indices(synth.rng(72, n), max(n, 1), ocodec.n_points, 48)
    lo = lo[:n]
    if n == 0:
        w = torch.full((3,), 7, dtype=torch.int64, device="cuda")
        gcodec.encode(torch.zeros((1, 24), dtype=torch.int8, device="cuda"), w, n=0)
        torch.cuda.synchronize()
        assert (w.cpu() == 7).all()
        return
    assert np.array_equal(gpu_encode(gcodec, ocodec.decode_batch(lo)), lo)


# ------------------------------------------------------------------ fused products ---------
def run_gemm(gcodec, layer, batch=None):
    import codebook_free_lattice_b200 as L
    batch = layer.batch if batch is None else batch
    words = torch.from_numpy(np.ascontiguousarray(layer.words).view(np.int64)).cuda()
    gains = torch.from_numpy(layer.gains.view(np.int16)).cuda()
    X = torch.from_numpy(layer.x[:batch].view(np.int16)).cuda()
    Y = torch.full((batch, layer.rows), float("nan"), dtype=torch.float32, device="cuda")
    w = gcodec.weight(words, gains, layer.rows, layer.K, layer.gain_mode, layer.pitch)
    if batch == 1:
        gcodec.gemv(w, X, Y)
    else:
        gcodec.gemm(w, X, Y, batch)
    torch.cuda.synchronize()
    assert gcodec.get_error() == 0
    return Y.cpu().numpy().astype(np.float64)


def oracle_gemm(ocodec, layer, rows=None, batch=None, threads=None):
    batch = layer.batch if batch is None else batch
    words = layer.words if rows is None else layer.words[rows]
    gains = layer.gains if rows is None else layer.gains[rows]
    return ocodec.gemm(words, layer.nb, layer.gain_mode, gains, layer.x[:batch], batch,
                       row_pitch_words=layer.pitch, threads=threads or (os.cpu_count() or 1))


def norms_from_oracle(ocodec):
    def fn(lo, hi):
        v = ocodec.decode_batch(lo).astype(np.float64)
        return np.sqrt((v ** 2).sum(1))
    return fn


def test_gemv_small_direct_gains(gcodec, ocodec):
    """240 x 384 (16 blocks per row), indices uniform over shells 2..4, direct fp16 gains."""
    layer = Layer(48, 240, 384, 1, 1, ocodec.n_points, 0, index_limit=415003680,
                  norms_fn=norms_from_oracle(ocodec))
    y = run_gemm(gcodec, layer)
    ref = oracle_gemm(ocodec, layer)
    assert max_rel_err(y, ref) < GEMV_RTOL


def test_gemv_one_hot_exact(gcodec, ocodec):
    """x = e_j with direct gains: y = g * v exactly (one product, exact in fp32)."""
    layer = Layer(48, 300, 24 * 7, 1, 4, ocodec.n_points, 0, norms_fn=norms_from_oracle(ocodec))
    for j in (0, 23, 24 * 7 - 1, 77):
        layer.x[:] = 0
        layer.x[0, j] = 1.0
        y = run_gemm(gcodec, layer)
        ref = oracle_gemm(ocodec, layer, threads=1)
        assert np.array_equal(y, ref)


@pytest.mark.parametrize("rows,K,batch,pitch", [(97, 1000, 1, None), (333, 24 * 37, 3, 40),
                                                (64, 4096, 8, None), (50, 2000, 16, None)])
def test_gemm_table_gains_ragged(gcodec, ocodec, rows, K, batch, pitch):
    layer = Layer(48, rows, K, batch, 5 + batch, ocodec.n_points, 1, pitch=pitch)
    y = run_gemm(gcodec, layer)
    ref = oracle_gemm(ocodec, layer)
    assert max_rel_err(y, ref) < GEMV_RTOL


@pytest.mark.parametrize("batch", [1, 3, 16])
def test_gemm_out_of_range_blocks(gcodec, ocodec, batch):
    """Blocks whose index is >= N_M contribute nothing (the oracle skips them) and raise the
    index-range flag, on the CUDA-core path (batch 1, 3) and the tensor-core path (batch 16)."""
    import codebook_free_lattice_b200 as L
    layer = Layer(48, 150, 24 * 37, batch, 30 + batch, ocodec.n_points, 1)
    w = layer.words.reshape(-1)
    w[::17] = (w[::17] & ~np.uint64(0xFFFFFFFFFFFF)) | np.uint64(ocodec.n_points + 99)
    w[5::23] = (w[5::23] & ~np.uint64(0xFFFFFFFFFFFF)) | np.uint64(2**48 - 1)
    words = torch.from_numpy(np.ascontiguousarray(layer.words).view(np.int64)).cuda()
    gains = torch.from_numpy(layer.gains.view(np.int16)).cuda()
    X = torch.from_numpy(layer.x[:batch].view(np.int16)).cuda()
    Y = torch.full((batch, layer.rows), float("nan"), dtype=torch.float32, device="cuda")
    wt = gcodec.weight(words, gains, layer.rows, layer.K, layer.gain_mode, layer.pitch)
    if batch == 1:
        gcodec.gemv(wt, X, Y)
    else:
        gcodec.gemm(wt, X, Y, batch)
    assert gcodec.get_error() == L.LLVQ_FLAG_INDEX_RANGE
    y = Y.cpu().numpy().astype(np.float64)
    assert max_rel_err(y, oracle_gemm(ocodec, layer)) < GEMV_RTOL


def test_gemm_batch_equals_gemv_columns(gcodec, ocodec):
    layer = Layer(48, 200, 24 * 50, 5, 9, ocodec.n_points, 1)
    Y = run_gemm(gcodec, layer)
    for b in range(5):
        sub = Layer(48, 200, 24 * 50, 5, 9, ocodec.n_points, 1)
        sub.x = layer.x[b:b + 1].copy()
        sub.batch = 1
        yb = run_gemm(gcodec, sub)
        # same decoded weights and products; only the fp32 summation order differs (blocks reach
        # the shared accumulators in an order fixed by atomics), hence a reassociation tolerance
        assert max_rel_err(yb[0], Y[b]) < 1e-4


@pytest.mark.parametrize("bits,rows,K", [(48, 300, 24 * 45 + 5), (72, 130, 24 * 9)])
def test_tensor_core_batch_equals_column_gemvs(gcodec, gcodec72, ocodec, ocodec72, bits, rows, K):
    """Batch 16 against 16 separate batch-1 products: at 48 bits the tensor-core path (ragged
    128-row tile and ragged 8-block round) against the coset-sorted GEMV, at 72 bits the 16-wide
    CUDA-core kernel against the batch-1 one."""
    g, o = (gcodec, ocodec) if bits == 48 else (gcodec72, ocodec72)
    layer = Layer(bits, rows, K, 16, 60 + bits, o.n_points, 1)
    Y = run_gemm(g, layer)
    for b in range(16):
        sub = Layer(bits, rows, K, 16, 60 + bits, o.n_points, 1)
        sub.x = layer.x[b:b + 1].copy()
        sub.batch = 1
        assert max_rel_err(run_gemm(g, sub)[0], Y[b]) < 1e-4
    assert max_rel_err(Y, oracle_gemm(o, layer)) < GEMV_RTOL


@pytest.mark.parametrize("rows,K,batch", [(4096, 4096, 1), (11008, 4096, 4), (4096, 11008, 1),
                                          (28672, 8192, 16)])
def test_gemm_full_size_sampled_rows(gcodec, ocodec, rows, K, batch):
    """Llama-2-7B layer shapes at the bench's launch configuration; the oracle checks a seeded
    sample of 256 rows."""
    layer = Layer(48, rows, K, batch, 20 + rows % 97, ocodec.n_points, 1)
    y = run_gemm(gcodec, layer)
    rs = np.sort(np.random.default_rng(rows + K).choice(rows, 256, replace=False))
    ref = oracle_gemm(ocodec, layer, rows=rs)
    assert max_rel_err(y[:, rs], ref) < GEMV_RTOL
    assert np.isfinite(y).all()


def test_argument_errors(gcodec):
    import codebook_free_lattice_b200 as L
    lib = L.lib()
    words = torch.zeros(64, dtype=torch.int64, device="cuda")
    out = torch.zeros(64 * 24 + 8, dtype=torch.int8, device="cuda")
    import ctypes as C
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.llvq_decode(gcodec.handle, C.c_void_p(words.data_ptr()), 16, 4, C.c_void_p(out.data_ptr()), s) == L.LLVQ_ERR_ARG
    assert lib.llvq_decode(gcodec.handle, C.c_void_p(words.data_ptr() + 4), 8, 4, C.c_void_p(out.data_ptr()), s) == L.LLVQ_ERR_ARG
    assert lib.llvq_decode(gcodec.handle, C.c_void_p(words.data_ptr()), 8, -1, C.c_void_p(out.data_ptr()), s) == L.LLVQ_ERR_ARG
    gains = torch.zeros(256 * 4, dtype=torch.int16, device="cuda")
    x = torch.zeros(24 * 4, dtype=torch.int16, device="cuda")
    y = torch.zeros(4 * 16, dtype=torch.float32, device="cuda")
    w = gcodec.weight(words, gains, 4, 96, 1)
    for batch in (0, 17):
        assert lib.llvq_gemm_smallbatch(gcodec.handle, C.byref(w), C.c_void_p(x.data_ptr()), batch,
                                        C.c_void_p(y.data_ptr()), s) == L.LLVQ_ERR_ARG
    bad = gcodec.weight(words, gains, 4, 96, 1)
    bad.blocks_per_row = 5
    assert lib.llvq_gemv(gcodec.handle, C.byref(bad), C.c_void_p(x.data_ptr()), C.c_void_p(y.data_ptr()), s) == L.LLVQ_ERR_ARG
    bad = gcodec.weight(words, gains, 4, 96, 1)
    bad.index_bits = 72
    assert lib.llvq_gemv(gcodec.handle, C.byref(bad), C.c_void_p(x.data_ptr()), C.c_void_p(y.data_ptr()), s) == L.LLVQ_ERR_ARG
    assert L.Codec(48).get_error() == 0


# ------------------------------------------------------------------ 72-bit budget ----------
def split128(vals):
    lo = np.array([v & (2**64 - 1) for v in vals], dtype=np.uint64)
    hi = np.array([v >> 64 for v in vals], dtype=np.uint64)
    return lo, hi


@pytest.mark.parametrize("batch", [8, 11])
def test_gemm72_cuda_core_batches(gcodec72, ocodec72, batch):
    """Batch 8 (its own instantiation) and batch 11 (the 16-wide kernel with a runtime batch) on
    the CUDA cores, ragged rows and blocks, against the oracle."""
    layer = Layer(72, 150, 24 * 21 + 5, batch, 90 + batch, ocodec72.n_points, 1)
    assert max_rel_err(run_gemm(gcodec72, layer), oracle_gemm(ocodec72, layer)) < GEMV_RTOL


def test_codec72_info_matches_oracle(gcodec72, ocodec72):
    assert gcodec72.max_shell == ocodec72.max_shell == 53
    assert gcodec72.n_points == ocodec72.n_points
    assert gcodec72.n_classes == 114976


def test_decode72_uniform(gcodec72, ocodec72):
    lo, hi = synth.uniform_indices(synth.rng(11, 0), 200_000, ocodec72.n_points, 72)
    codes = synth.gain_codes(synth.rng(11, 1), lo.shape[0])
    words = synth.pack_words(lo, hi, codes, 72)              # gain bits must be ignored
    got = gpu_decode(gcodec72, words)
    assert np.array_equal(got, ocodec72.decode_batch(lo, hi))
    assert gcodec72.get_error() == 0


def test_decode72_every_class(gcodec72, ocodec72):
    """First, middle and last index of all 114,976 classes (nine-group classes included) and
    all of shell 2."""
    idx = list(range(196560))
    for c in ocodec72.classes():
        idx += [c.offset, c.offset + c.size // 2, c.offset + c.size - 1]
    lo, hi = split128(idx)
    got = gpu_decode(gcodec72, synth.pack_words(lo, hi, None, 72))
    assert np.array_equal(got, ocodec72.decode_batch(lo, hi))


def test_decode72_out_of_range(gcodec72, ocodec72):
    N = ocodec72.n_points
    idx = [0, N - 1, N, N + 7, 2**72 - 1]
    lo, hi = split128(idx)
    got = gpu_decode(gcodec72, synth.pack_words(lo, hi, None, 72))
    assert gcodec72.get_error() == 1
    assert np.array_equal(got, ocodec72.decode_batch(lo, hi))
    assert (got[2:] == 0).all()


@pytest.mark.parametrize("rows,K,batch,mode", [(97, 1000, 1, 1), (64, 24 * 37, 4, 0), (40, 2000, 16, 1)])
def test_gemm72_ragged(gcodec72, ocodec72, rows, K, batch, mode):
    def norms(lo, hi):
        v = ocodec72.decode_batch(lo, hi).astype(np.float64)
        return np.sqrt((v ** 2).sum(1))
    layer = Layer(72, rows, K, batch, 30 + batch, ocodec72.n_points, mode, norms_fn=norms)
    y = run_gemm(gcodec72, layer)
    ref = oracle_gemm(ocodec72, layer)
    assert max_rel_err(y, ref) < GEMV_RTOL


@pytest.mark.parametrize("rows,K,batch", [(28672, 8192, 1), (8192, 28672, 8)])
def test_gemm72_full_size_sampled_rows(gcodec72, ocodec72, rows, K, batch):
    """Llama-2-70B layer shapes at 3 bits (72-bit indices in 16-byte words); 64 sampled rows."""
    layer = Layer(72, rows, K, batch, 40 + batch, ocodec72.n_points, 1)
    y = run_gemm(gcodec72, layer)
    rs = np.sort(np.random.default_rng(rows).choice(rows, 64, replace=False))
    ref = oracle_gemm(ocodec72, layer, rows=rs)
    assert max_rel_err(y[:, rs], ref) < GEMV_RTOL


def gpu_encode72(gcodec, vecs):
    v = torch.from_numpy(np.ascontiguousarray(vecs, np.int8)).cuda()
    w = torch.full((vecs.shape[0], 2), -1, dtype=torch.int64, device="cuda")
    gcodec.encode(v, w)
    torch.cuda.synchronize()
    out = w.cpu().numpy().view(np.uint64)
    return out[:, 0], out[:, 1]


def test_encode72_roundtrip_uniform_and_boundaries(gcodec72, ocodec72):
    """100,000 seeded uniform 72-bit indices and the first, middle and last index of every class,
    decoded by the oracle, encode back to themselves (gain bits zero)."""
    lo, hi = synth.uniform_indices(synth.rng(73, 0), 100_000, ocodec72.n_points, 72)
    b_lo, b_hi = [], []
    for c in ocodec72.classes():
        for i in (c.offset, c.offset + c.size // 2, c.offset + c.size - 1):
            b_lo.append(i & (2**64 - 1))
            b_hi.append(i >> 64)
    lo = np.concatenate([lo, np.array(b_lo, np.uint64)])
    hi = np.concatenate([hi, np.array(b_hi, np.uint64)])
    vecs = ocodec72.decode_batch(lo, hi)
    glo, ghi = gpu_encode72(gcodec72, vecs)
    assert np.array_equal(glo, lo) and np.array_equal(ghi, hi)
    assert gcodec72.get_error() == 0
    for t in range(0, 100_000, 997):
        assert (int(ghi[t]) << 64 | int(glo[t])) == ocodec72.encode(vecs[t].astype(np.int32))


def test_encode72_not_coded(gcodec72, ocodec72):
    lo, hi = synth.uniform_indices(synth.rng(74, 0), 16, ocodec72.n_points, 72)
    good = ocodec72.decode_batch(lo, hi)
    v1 = good[0].copy(); v1[2] += 2                                   # breaks the congruences
    v2 = good[1].copy(); v2[7] ^= 1                                   # mixed parity
    bad = np.stack([np.zeros(24, np.int8), v1, v2])
    for b_ in bad:
        with pytest.raises(ValueError):
            ocodec72.encode(b_.astype(np.int32))
    glo, ghi = gpu_encode72(gcodec72, np.concatenate([good, bad]))
    assert gcodec72.get_error() == 4
    assert np.array_equal(glo[:16], lo) and np.array_equal(ghi[:16], hi)
    assert (glo[16:] == np.uint64(2**64 - 1)).all() and (ghi[16:] == 0xFF).all()




# ------------------------------------------------------------------ 96-bit budget ----------
# The oracle builds the class list of a 96-bit shell on demand (up to 9.1M classes for shell
# 214) and decodes in ascending index order, so the cases below draw their indices from a few
# shells each.

@pytest.fixture(scope="module")
def gcodec96(dev):
    import codebook_free_lattice_b200 as L
    return L.Codec(96)


@pytest.fixture(scope="module")
def ocodec96():
    return oracle.Codec(96)


def split96(idx):
    lo = np.array([i & (2**64 - 1) for i in idx], np.uint64)
    hi = np.array([i >> 64 for i in idx], np.uint64)
    return lo, hi


def uniform_in_shells(ocodec, m0, m1, n, seed):
    """n seeded indices uniform over shells m0..m1 (python ints)."""
    a, b = ocodec.shell_offset(m0), ocodec.shell_offset(m1 + 1)
    lo, hi = synth.uniform_indices(synth.rng(seed, 0), n, b - a, 96)
    return [a + (int(h) << 64 | int(l)) for l, h in zip(lo, hi)]


def test_codec96_info_matches_oracle(gcodec96, ocodec96):
    assert gcodec96.max_shell == ocodec96.max_shell == 214
    assert gcodec96.n_points == ocodec96.n_points == 74972166705387133681638419280
    assert gcodec96.n_classes == 304649365


def test_decode96_class_boundaries_and_shells(gcodec96, ocodec96):
    """First, middle and last index of every class of shells 2..9 and of sampled classes of
    shells 50, 120, 200 and 214; seeded uniform indices inside shells 3, 50, 120, 200 and 214;
    the last coded index.  Gain-code bits must be ignored."""
    idx = []
    for m in range(2, 10):
        for j in range(ocodec96.shell_nclasses(m)):
            c = ocodec96.shell_class(m, j)
            idx += [c.offset, c.offset + c.size // 2, c.offset + c.size - 1]
    for m in (50, 120, 200, 214):
        n = ocodec96.shell_nclasses(m)
        for j in list(range(0, n, max(1, n // 150))) + [n - 1]:
            c = ocodec96.shell_class(m, j)
            idx += [c.offset, c.offset + c.size - 1]
    for seed, m in enumerate((3, 50, 120, 200, 214)):
        idx += uniform_in_shells(ocodec96, m, m, 400, 40 + seed)
    idx.append(ocodec96.n_points - 1)
    lo, hi = split96(idx)
    codes = synth.gain_codes(synth.rng(45, 1), lo.shape[0])
    got = gpu_decode(gcodec96, synth.pack_words(lo, hi, codes, 96))
    assert np.array_equal(got, ocodec96.decode_batch(lo, hi))
    assert gcodec96.get_error() == 0


def test_decode96_top_shells_uniform(gcodec96, ocodec96):
    """6000 seeded indices uniform over shells 205..214, which hold 38% of the index space."""
    lo, hi = split96(uniform_in_shells(ocodec96, 205, 214, 6000, 46))
    got = gpu_decode(gcodec96, synth.pack_words(lo, hi, None, 96))
    assert np.array_equal(got, ocodec96.decode_batch(lo, hi))


def test_decode96_out_of_range(gcodec96, ocodec96):
    N = ocodec96.n_points
    lo, hi = split96([0, N - 1, N, N + 7, 2**96 - 1, 5])
    got = gpu_decode(gcodec96, synth.pack_words(lo, hi, None, 96))
    assert gcodec96.get_error() == 1
    assert np.array_equal(got, ocodec96.decode_batch(lo, hi))
    assert (got[2:5] == 0).all()


@pytest.mark.parametrize("batch,rows,K,gain_mode", [(1, 150, 24 * 33 + 7, 1), (3, 70, 24 * 20, 0),
                                                    (16, 200, 24 * 13, 1)])
def test_gemm96_low_shells(gcodec96, ocodec96, batch, rows, K, gain_mode):
    """GEMV, CUDA-core batch 3 and tensor-core batch 16 on indices uniform over shells 2..60."""
    limit = ocodec96.shell_offset(61)
    norms = None
    if gain_mode == 0:
        def norms(lo, hi):
            v = ocodec96.decode_batch(lo, hi).astype(np.float64)
            return np.sqrt((v ** 2).sum(1))
    layer = Layer(96, rows, K, batch, 50 + batch, ocodec96.n_points, gain_mode, index_limit=limit,
                  norms_fn=norms)
    y = run_gemm(gcodec96, layer)
    assert max_rel_err(y, oracle_gemm(ocodec96, layer)) < GEMV_RTOL


@pytest.mark.parametrize("batch", [8, 13])
def test_gemm96_cuda_core_batches(gcodec96, ocodec96, batch):
    """Batch 8 and batch 13 (runtime batch in the 16-wide kernel), indices over shells 2..60."""
    layer = Layer(96, 90, 24 * 17 + 3, batch, 95 + batch, ocodec96.n_points, 1,
                  index_limit=ocodec96.shell_offset(61))
    assert max_rel_err(run_gemm(gcodec96, layer), oracle_gemm(ocodec96, layer)) < GEMV_RTOL


@pytest.mark.parametrize("batch", [1, 16])
def test_gemm96_top_shells(gcodec96, ocodec96, batch):
    """Products on indices uniform over shells 208..214 (u8 gain tables)."""
    layer = Layer(96, 64, 24 * 40, batch, 60 + batch, ocodec96.n_points, 1,
                  index_base=ocodec96.shell_offset(208))
    y = run_gemm(gcodec96, layer)
    assert max_rel_err(y, oracle_gemm(ocodec96, layer)) < GEMV_RTOL


def test_encode96_roundtrip(gcodec96, ocodec96):
    """Every class boundary of shells 2..6, sampled classes of shells 120 and 214, seeded uniform
    indices inside shells 3, 50 and 214 and over shells 205..214, and the last coded index:
    decoded by the oracle, they encode back to themselves; a sample also equals the oracle's
    encode."""
    idx = []
    for m in range(2, 7):
        for j in range(ocodec96.shell_nclasses(m)):
            c = ocodec96.shell_class(m, j)
            idx += [c.offset, c.offset + c.size // 2, c.offset + c.size - 1]
    for m in (120, 214):
        n = ocodec96.shell_nclasses(m)
        for j in list(range(0, n, max(1, n // 60))) + [n - 1]:
            c = ocodec96.shell_class(m, j)
            idx += [c.offset, c.offset + c.size - 1]
    for seed, m in enumerate((3, 50, 214)):
        idx += uniform_in_shells(ocodec96, m, m, 300, 80 + seed)
    idx += uniform_in_shells(ocodec96, 205, 214, 2000, 84)
    idx.append(ocodec96.n_points - 1)
    lo, hi = split96(idx)
    vecs = ocodec96.decode_batch(lo, hi)
    glo, ghi = gpu_encode72(gcodec96, vecs)
    assert np.array_equal(glo, lo) and np.array_equal(ghi, hi)
    assert gcodec96.get_error() == 0
    for t in range(0, len(idx), 97):
        assert (int(ghi[t]) << 64 | int(glo[t])) == ocodec96.encode(vecs[t].astype(np.int32))


def test_encode96_not_coded(gcodec96, ocodec96):
    lo, hi = split96(uniform_in_shells(ocodec96, 2, 40, 16, 85))
    good = ocodec96.decode_batch(lo, hi)
    v1 = good[0].copy(); v1[2] += 2                                   # breaks the congruences
    v2 = good[1].copy(); v2[7] ^= 1                                   # mixed parity
    big = (ocodec96.decode_batch(np.array([98256], np.uint64))[0] * 12).astype(np.int8)   # shell 288 > 214
    bad = np.stack([np.zeros(24, np.int8), v1, v2, big])
    for b_ in bad:
        with pytest.raises(ValueError):
            ocodec96.encode(b_.astype(np.int32))
    glo, ghi = gpu_encode72(gcodec96, np.concatenate([good, bad]))
    assert gcodec96.get_error() == 4
    assert np.array_equal(glo[:16], lo) and np.array_equal(ghi[:16], hi)
    assert (glo[16:] == np.uint64(2**64 - 1)).all() and (ghi[16:] == 0xFFFFFFFF).all()
