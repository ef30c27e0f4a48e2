"""Host-built class records of the 96-bit budget (what the 96-bit decoder reads from global
memory) against the oracle's class lists, on the CPU.

Each record must carry its class's first index, shell, coset, codeword weight k, free sign bits
B, parity target, the cumulative counts and magnitudes of its groups in the decoder's order
(even coset: magnitudes 0 mod 4 ascending, then 2 mod 4 ascending; odd: all ascending), and the
reciprocal ceil(2^(128+t)/P) - 2^128 of its arrangement count P (t = bitlen(P - 1)).  Consecutive
starts must differ by the class size A 2^B P, with P recomputed here as a multinomial of the
group counts (papernotes.org notes, 关键设计 2: contiguous class ranges, I_class = r + A (s + 2^B p)).
"""
import math

import numpy as np
import pytest

import oracle

L = pytest.importorskip("codebook_free_lattice_b200")


@pytest.fixture(scope="module")
def o96():
    return oracle.Codec(96)


def groups_in_decoder_order(c):
    pairs = list(zip(c.vals, c.cnts))
    if c.odd:
        return sorted(pairs)
    return sorted(p for p in pairs if p[0] % 4 == 0) + sorted(p for p in pairs if p[0] % 4 == 2)


def multinomial(counts):
    n = sum(counts)
    r = math.factorial(n)
    for k in counts:
        r //= math.factorial(k)
    return r


def check_record(rec, c, m):
    start = int(rec["start_lo"]) | int(rec["start_hi"]) << 64
    meta = int(rec["meta"])
    assert start == c.offset
    assert (meta >> 7) & 0xFF == m
    assert bool(meta >> 25 & 1) == c.odd
    assert (meta >> 20) & 0x1F == c.B
    if not c.odd:
        assert (meta >> 15) & 0x1F == c.k
        assert meta >> 26 & 1 == (sum(v * n for v, n in zip(c.vals, c.cnts)) // 4) & 1
    order = groups_in_decoder_order(c)
    cum = 0
    for g in range(16):
        if g < len(order):
            cum += order[g][1]
            assert rec["cum"][g] == 0x7F + cum and rec["vals"][g] == order[g][0]
        else:
            assert rec["cum"][g] == 0x7F + 24 and rec["vals"][g] == 0
    t = (c.P - 1).bit_length()
    assert meta & 0x7F == t
    rcp = int(rec["rcp_lo"]) | int(rec["rcp_hi"]) << 64
    assert rcp == -(-(2 ** (128 + t)) // c.P) - 2 ** 128


@pytest.mark.parametrize("m", [2, 3, 4, 5, 6, 7, 8, 20, 50])
def test_every_record_of_small_shells(o96, m):
    recs = L.class_table96(m)
    assert len(recs) == o96.shell_nclasses(m)
    for j in range(len(recs)):
        check_record(recs[j], o96.shell_class(m, j), m)


@pytest.mark.parametrize("m", [120, 214])
def test_sampled_records_and_contiguous_sizes(o96, m):
    recs = L.class_table96(m)
    n = o96.shell_nclasses(m)
    assert len(recs) == n
    for j in list(range(0, n, max(1, n // 300))) + [n - 1]:
        check_record(recs[j], o96.shell_class(m, j), m)
    # consecutive starts differ by A 2^B P, with P from the recorded group counts
    starts = [int(r["start_lo"]) | int(r["start_hi"]) << 64 for r in recs[:2000]]
    for j in range(len(starts) - 1):
        r = recs[j]
        cum = [int(x) - 0x7F for x in r["cum"]]
        cnt = [cum[0]] + [cum[g] - cum[g - 1] for g in range(1, 16)]
        meta = int(r["meta"])
        odd, k, B = bool(meta >> 25 & 1), (meta >> 15) & 0x1F, (meta >> 20) & 0x1F
        if odd:
            A, P = 4096, multinomial([x for x in cnt if x])
        else:
            vals = [int(v) for v in r["vals"]]
            off = [cnt[g] for g in range(16) if cnt[g] and vals[g] % 4 == 0]
            on = [cnt[g] for g in range(16) if cnt[g] and vals[g] % 4 == 2]
            A, P = {0: 1, 8: 759, 12: 2576, 16: 759, 24: 1}[k], multinomial(off) * multinomial(on)
        assert starts[j + 1] - starts[j] == A * 2 ** B * P
    assert starts[0] == o96.shell_offset(m)


def test_shell_range_and_errors():
    import ctypes as C
    n = C.c_int64()
    assert L.lib().llvq_class_table96(1, None, 0, C.byref(n)) == L.LLVQ_ERR_ARG
    assert L.lib().llvq_class_table96(215, None, 0, C.byref(n)) == L.LLVQ_ERR_ARG
    assert L.lib().llvq_class_table96(214, None, 0, C.byref(n)) == L.LLVQ_OK and n.value == 9124194
    small = (L.llvq_class96 * 2)()
    assert L.lib().llvq_class_table96(4, C.cast(small, C.c_void_p), 2, C.byref(n)) == L.LLVQ_ERR_ARG


def test_shell_starts_match_theta_series():
    """Shell m's class records span exactly N_m indices, N_m from the theta series computed here
    independently (tests/theta.py, Python integers), for m = 2..40."""
    from tests.theta import leech_shell_sizes
    N = leech_shell_sizes(41)
    starts = {}
    for m in range(2, 42):
        r0 = L.class_table96(m)[0]
        starts[m] = int(r0["start_lo"]) | int(r0["start_hi"]) << 64
    assert starts[2] == 0
    for m in range(2, 41):
        assert starts[m + 1] - starts[m] == N[m], m

