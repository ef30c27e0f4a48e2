"""CPU check of the search kernel's compile-time class table (csrc/search48_classes.cuh).

The header is plain constexpr C++, so it compiles with the host compiler: a small program prints
every class, and the list must equal the oracle's class list of the 48-bit union in index order
(shell, coset, magnitude multiset), with the column entries, steps, sign parity and sign-turn cost
that the search's closed form needs derived here from the oracle's multisets:
  kinds: odd 1 / 3 (mod 4), even 2 (mod 4) on S / 0 (mod 4) off S, zeros dropped; each kind in
  descending magnitude; entry = 25 * kind + (count of that kind's magnitudes >= a); step =
  a - (next smaller magnitude of the kind, 0 after the last); even parity = (sum / 4) mod 2 when
  k > 0; turn cost = 2 x the smallest 2-mod-4 magnitude.
(The codec repeats this comparison against its own host tables when it is created.)
A second check compiles the host helper that gives, per class list, the prefix lying in shells
2..M (the search skips the rest), and compares it with the oracle's class counts.
"""
import os
import shutil
import subprocess

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "codebook_free_lattice_b200", "csrc")

PROGRAM = r'''
#include "search48_classes.cuh"
#include <cstdio>
int main() {
    const auto &T = llvq::search_cx::kTable;
    std::printf("%d %d", T.n, T.n_odd);
    for (int w = 0; w < 5; w++) std::printf(" %d", T.n_even[w]);
    std::printf("\n");
    for (int i = 0; i < T.n; i++) {
        const auto &c = T.c[i];
        std::printf("%d %d %d %d %d %d |", c.id, c.m, c.odd, c.k, c.q, c.turn2);
        for (int j = 0; j < c.nv; j++) std::printf(" %d:%d", c.val[j], c.cnt[j]);
        std::printf(" |");
        for (int g = 0; g < c.ng; g++) std::printf(" %d/%d", c.e[g], c.da[g]);
        std::printf("\n");
    }
}
'''


def derive(c):
    """(groups, parity, turn cost) of an oracle class, by the rules in the module docstring."""
    vc = sorted(zip(c.vals, c.cnts), reverse=True)
    groups = []
    for kind in (0, 1):
        mags = [(a, n) for a, n in vc if a != 0 and ((a % 4 == 3) if c.odd else (a % 4 == 0)) == bool(kind)]
        cum = 0
        for u, (a, n) in enumerate(mags):
            cum += n
            nxt = mags[u + 1][0] if u + 1 < len(mags) else 0
            groups.append((25 * kind + cum, a - nxt))
    k = 0 if c.odd else c.k
    q = (sum(a * n for a, n in vc) // 4) & 1 if (not c.odd and k > 0) else 0
    on_s = [a for a, n in vc if a % 4 == 2]
    turn2 = 2 * min(on_s) if (not c.odd and on_s) else 0
    return groups, q, turn2


def test_compile_time_table_equals_the_oracle_classes(tmp_path):
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    src = tmp_path / "dump.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "dump"
    subprocess.run([cxx, "-std=c++17", "-O1", "-I", CSRC, "-o", str(exe), str(src)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines()
    head = list(map(int, out[0].split()))
    o = oracle.Codec(48)
    classes = list(o.classes())
    by_weight = [sum(1 for c in classes if not c.odd and c.k == w) for w in (0, 8, 12, 16, 24)]
    assert head == [len(classes), sum(c.odd for c in classes)] + by_weight == [383, 157, 17, 86, 68, 50, 5]
    for i, (line, c) in enumerate(zip(out[1:], classes)):
        meta, mult, grp = line.split("|")
        cid, m, odd, k, q, turn2 = map(int, meta.split())
        assert (cid, m, odd) == (i, c.m, int(c.odd))
        assert mult.split() == [f"{a}:{n}" for a, n in sorted(zip(c.vals, c.cnts), reverse=True)]
        groups, q_ref, t_ref = derive(c)
        assert [tuple(map(int, g.split("/"))) for g in grp.split()] == groups, i
        assert (q, turn2) == (q_ref, t_ref), i
        if not c.odd:
            assert k == c.k


PREFIX_PROGRAM = r'''
#include "search48.cuh"
#include <cstdio>
int main() {
    for (int ms = 2; ms <= 13; ms++) {
        int nal[6];
        llvq::search_list_prefixes(ms, nal);
        std::printf("%d", ms);
        for (int l = 0; l < 6; l++) std::printf(" %d", nal[l]);
        std::printf("\n");
    }
}
'''


def test_union_is_a_prefix_of_each_class_list(tmp_path):
    """A search over shells 2..M skips, in each class list (odd; even by codeword weight), the
    classes past a prefix; the prefix lengths the host computes must be the numbers of classes of
    shells <= M in that list (so each list must be in shell order)."""
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("no nvcc")
    src = tmp_path / "prefix.cu"
    src.write_text(PREFIX_PROGRAM)
    exe = tmp_path / "prefix"
    subprocess.run([nvcc, "-std=c++17", "--expt-relaxed-constexpr", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", CSRC, "-o", str(exe), str(src)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines()
    classes = list(oracle.Codec(48).classes())
    lists = [[c for c in classes if c.odd]] + [[c for c in classes if not c.odd and c.k == w] for w in (0, 8, 12, 16, 24)]
    for line in out:
        ms, *nal = map(int, line.split())
        assert nal == [sum(1 for c in L if c.m <= ms) for L in lists], ms
    for L in lists:
        assert [c.m for c in L] == sorted(c.m for c in L)
