"""CPU pins of the facts the GPU encoders rely on, checked against the oracle's Golay code and
class lists (papernotes.org notes, 关键设计 2: classes are contiguous ranges ordered inside a
shell; the codeword index r counts codewords in a fixed order).

- Coordinates 12..23 are an information set of the code: codeword t in ascending mask order has
  top 12 bits t, so a codeword's place is read from its top 12 bits.
- Inside one (shell, coset), the classes ascend by the keys the encoders search:
  48-bit: counts of |x| = 0..13, 5 bits each, the largest magnitude most significant;
  72/96-bit: the unary code of the counts read from the largest magnitude of the coset down
  ("count ones, then a zero"), 39 bits at 72 and 54 bits at 96 bits.
"""
import numpy as np
import pytest

import oracle


def count_key48(c):
    key = 0
    for v, n in zip(c.vals, c.cnts):
        key += n << (5 * v)
    return key


def unary_key(c, top):
    cnt = {v: n for v, n in zip(c.vals, c.cnts)}
    key, bits = 0, 0
    for v in range(top, -1, -2):                 # the coset's magnitudes, largest first
        n = cnt.get(v, 0)
        key = (key << (n + 1)) | (((1 << n) - 1) << 1)
        bits += n + 1
    return key, bits


def test_top12_information_set():
    w = oracle.golay_by_mask()
    assert np.array_equal(w >> 12, np.arange(4096, dtype=w.dtype))


def check_segments(classes, keyfn):
    seen = {}
    for c in classes:
        k = keyfn(c)
        seg = (c.m, c.odd)
        if seg in seen:
            assert seen[seg] < k, (c.m, c.odd, c.vals, c.cnts)
        seen[seg] = k
    return len(seen)


def test_48bit_count_keys_ascend():
    o = oracle.Codec(48)
    assert check_segments(o.classes(), count_key48) == 2 * 12
    assert max(v for c in o.classes() for v in c.vals) == 13


def test_72bit_unary_keys_ascend():
    o = oracle.Codec(72)
    assert max(v for c in o.classes() for v in c.vals) <= 29

    def key(c):
        k, bits = unary_key(c, 29 if c.odd else 28)
        assert bits == 39
        return k
    assert check_segments(o.classes(), key) == 2 * 52


@pytest.mark.parametrize("m", [2, 7, 60, 130])
def test_96bit_unary_keys_ascend_in_64_bits(m):
    o = oracle.Codec(96)
    cls = [o.shell_class(m, j) for j in range(o.shell_nclasses(m))]
    assert max(v for c in cls for v in c.vals) <= 58

    def key(c):
        k, bits = unary_key(c, 57 if c.odd else 58)
        assert bits == 24 + (29 if c.odd else 30) <= 64
        return k
    check_segments(cls, key)
