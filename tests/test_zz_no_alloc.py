"""The decode entry point that allocates no device memory (llvq_decode_noalloc).

Some callers cannot call cudaMalloc: a plug-in whose device memory all belongs to a framework's
caching allocator, or a latency-critical path where cudaMalloc's implicit device synchronisation
is not allowed.  For them the library keeps the 48-bit decode tables in a static device array
instead of a codec.  That entry point runs its own kernel (the plain one-thread-per-block decode
on the static tables), so it is checked here against the CPU oracle, element by element, on two
calls in a row: the first over shell 2, every class boundary and uniform indices; the second over
other indices, a ragged size and out-of-range indices (zero rows).  It is also checked against
llvq_decode, and device memory must not shrink across the calls after set-up.  This file is
collected last so that a failure here never hides the other tests.
"""
import ctypes as C

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _noalloc(lib, words_np):
    import codebook_free_lattice_b200 as L
    n = words_np.shape[0]
    w = torch.from_numpy(words_np.view(np.int64)).cuda()
    got = torch.full((n, 24), 99, dtype=torch.int8, device="cuda")
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.llvq_decode_noalloc(48, C.c_void_p(w.data_ptr()), 8, n, C.c_void_p(got.data_ptr()), s) == L.LLVQ_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    return got.cpu().numpy(), free0, free1


def test_noalloc_decode_matches_oracle_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import codebook_free_lattice_b200 as L
    import oracle
    from codebook_free_lattice_b200 import synth
    lib = L.lib()
    o = oracle.Codec(48)
    # set-up call (tables copied into the static array once per device)
    warm, _, _ = _noalloc(lib, np.arange(64, dtype=np.uint64))
    assert np.array_equal(warm, o.decode_batch(np.arange(64, dtype=np.uint64)))
    # first call: shell 2 in full, the first, middle and last index of every class, uniform
    # indices over the whole budget; gain bits set (they must be ignored)
    bounds = []
    for c in o.classes():
        bounds += [c.offset, c.offset + c.size // 2, c.offset + c.size - 1]
    lo, _ = synth.uniform_indices(synth.rng(91, 0), 100_000, o.n_points, 48)
    idx = np.concatenate([np.arange(196560, dtype=np.uint64), np.array(bounds, dtype=np.uint64), lo])
    words = synth.pack_words(idx, None, synth.gain_codes(synth.rng(91, 1), idx.shape[0]), 48)
    got, free0, free1 = _noalloc(lib, words)
    assert np.array_equal(got, o.decode_batch(idx))
    assert free1 >= free0                                   # nothing allocated on the device
    # second call: other indices, a ragged size and out-of-range indices (zero rows)
    lo2, _ = synth.uniform_indices(synth.rng(92, 0), 77_777, o.n_points, 48)
    bad = np.zeros(lo2.shape[0], dtype=bool)
    bad[::1000] = True
    lo2[bad] = np.uint64(o.n_points + 5)
    got2, free2, free3 = _noalloc(lib, lo2)
    assert (got2[bad] == 0).all()
    assert np.array_equal(got2[~bad], o.decode_batch(lo2[~bad]))
    assert free3 >= free2
    # the codec's decode agrees with it on the same words
    codec = L.Codec(48)
    w = torch.from_numpy(lo2.view(np.int64)).cuda()
    ref = torch.empty((lo2.shape[0], 24), dtype=torch.int8, device="cuda")
    codec.decode(w, ref)
    torch.cuda.synchronize()
    assert np.array_equal(ref.cpu().numpy(), got2)


def test_noalloc_rejects_other_budgets():
    import codebook_free_lattice_b200 as L
    lib = L.lib()
    assert lib.llvq_decode_noalloc(72, None, 16, 1, None, None) == L.LLVQ_ERR_UNSUPPORTED
    assert lib.llvq_decode_noalloc(48, None, 16, 1, None, None) == L.LLVQ_ERR_ARG
    assert lib.llvq_decode_noalloc(48, None, 8, -1, None, None) == L.LLVQ_ERR_ARG
