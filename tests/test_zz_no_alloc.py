"""The decode entry point that allocates no device memory (llvq_decode_noalloc).

It exists for callers that cannot call cudaMalloc (inside a CUDA-graph capture, or under a
framework allocator that owns the device memory): its tables live in a static device array in
the library instead of a codec.  It must agree bit for bit with llvq_decode, call after call,
because both run the same decode on the same tables.  This file is collected last so that a
failure here never hides the other tests.
"""
import ctypes as C

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _decode_both(lib, codec, words_np):
    import codebook_free_lattice_b200 as L
    n = words_np.shape[0]
    w = torch.from_numpy(words_np.view(np.int64)).cuda()
    ref = torch.empty((n, 24), dtype=torch.int8, device="cuda")
    got = torch.full((n, 24), 99, dtype=torch.int8, device="cuda")
    codec.decode(w, ref)
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.llvq_decode_noalloc(48, C.c_void_p(w.data_ptr()), 8, n, C.c_void_p(got.data_ptr()), s) == L.LLVQ_OK
    torch.cuda.synchronize()
    return got.cpu().numpy(), ref.cpu().numpy()


def test_noalloc_decode_matches_codec_decode_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from codebook_free_lattice_b200 import build, synth
    build.build()
    import codebook_free_lattice_b200 as L
    lib = L.lib()
    codec = L.Codec(48)
    # first call: shell 2 in full plus uniform indices, with gain bits set
    lo, _ = synth.uniform_indices(synth.rng(91, 0), 100_000, codec.n_points, 48)
    idx = np.concatenate([np.arange(196560, dtype=np.uint64), lo])
    words = synth.pack_words(idx, None, synth.gain_codes(synth.rng(91, 1), idx.shape[0]), 48)
    got, ref = _decode_both(lib, codec, words)
    assert np.array_equal(got, ref)
    # second call: other indices, a ragged size and out-of-range indices (zero rows)
    lo2, _ = synth.uniform_indices(synth.rng(92, 0), 77_777, codec.n_points, 48)
    lo2[::1000] = np.uint64(codec.n_points + 5)
    got2, ref2 = _decode_both(lib, codec, lo2)
    assert np.array_equal(got2, ref2)
    assert (got2[::1000] == 0).all()
    assert codec.get_error() == L.LLVQ_FLAG_INDEX_RANGE    # only the codec call raises the codec's flag


def test_noalloc_rejects_other_budgets():
    import codebook_free_lattice_b200 as L
    lib = L.lib()
    assert lib.llvq_decode_noalloc(72, None, 16, 1, None, None) == L.LLVQ_ERR_UNSUPPORTED
    assert lib.llvq_decode_noalloc(48, None, 16, 1, None, None) == L.LLVQ_ERR_ARG
    assert lib.llvq_decode_noalloc(48, None, 8, -1, None, None) == L.LLVQ_ERR_ARG
