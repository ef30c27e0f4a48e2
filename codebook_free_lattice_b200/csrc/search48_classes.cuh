// search48_classes.cuh -- the 383 classes of the 48-bit shell union (shells 2..13), built at
// compile time for the nearest-point search kernel, in the codec's index order.
//
// A class is a multiset of 24 magnitudes of one parity with sum of squares 16 m, in the even or
// odd coset ("Leech Lattice Vector Quantization for Efficient LLM Compression", papernotes.org
// notes, 方法详解 / 关键设计 2: classes are magnitude multisets with their coset, taking
// contiguous index ranges; gist.science, Methodik 1 and 3).  Admissible multisets: even -- the
// number k of magnitudes = 2 (mod 4) is a Golay codeword weight (0, 8, 12, 16, 24), and for k = 0
// the sum of magnitudes / 4 is even (a coordinate sum of 0 mod 8 must be reachable); odd -- the
// sum of (a if a = 3 mod 4 else -a) is 4 mod 8.  Order: shell ascending; even coset first; inside
// a coset, the magnitudes sorted descending, compared lexicographically ascending.  A depth-first
// walk over the magnitudes from the largest down, taking each magnitude's count in ascending
// order, visits the multisets in exactly that order.
//
// For the search each class also carries its column offsets and steps: the nonzero magnitudes
// split into two kinds (odd: 1 / 3 mod 4; even: 2 mod 4 on the codeword S / 0 mod 4 off S), each
// kind in descending order; group g of kind t reads column entry e_g = 25 t + (how many of that
// kind's magnitudes are >= a_g) with step da_g = a_g - (the next smaller magnitude of the kind,
// 0 after the last).  The codec checks this table against its own class list when it is created.
#pragma once

namespace llvq {
namespace search_cx {

constexpr int kShells = 13;           // the 48-bit union: shells 2..13
constexpr int kClasses = 383;
constexpr int kGroups = 5;            // nonzero magnitude groups a class can have
constexpr int kCols = 25;             // entries per kind: counts 0..24
constexpr int kWeights[5] = {0, 8, 12, 16, 24};

struct Cls {
    int m = 0, odd = 0, k = 0, id = 0;
    int nv = 0;                       // distinct magnitudes, descending
    int val[8] = {}, cnt[8] = {};
    int ng = 0;                       // nonzero groups
    int e[kGroups] = {};              // column entries
    int da[kGroups] = {};             // steps
    int q = 0;                        // even: parity of the negative signs the class needs on S
    int turn2 = 0;                    // even, k > 0: 2 x the smallest 2-mod-4 magnitude
};

struct Table {
    Cls c[kClasses] = {};
    int n = 0;
    int n_odd = 0;
    int odd_ids[kClasses] = {};
    int n_even[5] = {};
    int even_ids[5][kClasses] = {};
    bool overflow = false;
};

constexpr void add_class(Table &T, int m, int odd, const int (&vals)[16], const int (&cnt)[16], int nvals) {
    Cls c;
    c.m = m;
    c.odd = odd;
    int k = 0, sum_abs = 0, signed_sum = 0;
    for (int i = 0; i < nvals; i++) {
        if (cnt[i] == 0) continue;
        const int v = vals[i], n = cnt[i];
        c.val[c.nv] = v;
        c.cnt[c.nv] = n;
        c.nv++;
        if (v % 4 == 2) k += n;
        sum_abs += v * n;
        signed_sum += (v % 4 == 3 ? v : -v) * n;
    }
    if (odd) {
        if (((signed_sum % 8) + 8) % 8 != 4) return;
    } else {
        bool weight = false;
        for (int w : kWeights) weight = weight || w == k;
        if (!weight) return;
        if (k == 0 && (sum_abs / 4) % 2 != 0) return;
        c.k = k;
        c.q = k > 0 ? (sum_abs / 4) & 1 : 0;
    }
    // groups: kind 0 then kind 1, each descending (val[] is descending already)
    for (int kind = 0; kind < 2; kind++) {
        int cum = 0, last = -1;
        for (int i = 0; i < c.nv; i++) {
            const int v = c.val[i];
            if (v == 0) continue;
            const int kd = odd ? (v % 4 == 3) : (v % 4 == 0);
            if (kd != kind) continue;
            if (c.ng >= kGroups) { T.overflow = true; return; }
            cum += c.cnt[i];
            if (last >= 0) c.da[last] -= v;         // previous group's step: a_prev - a
            c.e[c.ng] = kind * kCols + cum;
            c.da[c.ng] = v;
            last = c.ng;
            c.ng++;
            if (!odd && kind == 0) c.turn2 = 2 * v;  // ends at the smallest 2-mod-4 magnitude
        }
    }
    if (T.n >= kClasses) { T.overflow = true; return; }
    c.id = T.n;
    if (odd) {
        T.odd_ids[T.n_odd++] = T.n;
    } else {
        for (int w = 0; w < 5; w++)
            if (kWeights[w] == k) T.even_ids[w][T.n_even[w]++] = T.n;
    }
    T.c[T.n++] = c;
}

// magnitudes vals[vi..] (descending) for `left` coordinates with squared norm `norm`
constexpr void walk(Table &T, int m, int odd, const int (&vals)[16], int nvals, int (&cnt)[16], int vi, int left,
                    int norm) {
    if (vi == nvals) {
        if (left == 0 && norm == 0) add_class(T, m, odd, vals, cnt, nvals);
        return;
    }
    const int v = vals[vi], sq = v * v;
    int maxn = left;
    if (sq > 0 && norm / sq < maxn) maxn = norm / sq;
    for (int n = 0; n <= maxn; n++) {
        const int rest = norm - n * sq, rest_left = left - n;
        if (vi + 1 < nvals) {
            const int vn = vals[vi + 1];
            if (rest_left * vn * vn < rest) continue;            // the smaller ones cannot absorb it
        } else if (rest != 0 || rest_left != 0) {
            continue;
        }
        cnt[vi] = n;
        walk(T, m, odd, vals, nvals, cnt, vi + 1, rest_left, rest);
        cnt[vi] = 0;
    }
}

constexpr Table make_table() {
    Table T;
    for (int m = 2; m <= kShells; m++) {
        for (int odd = 0; odd <= 1; odd++) {
            int vals[16] = {}, cnt[16] = {}, nvals = 0;
            for (int v = 15; v >= 0; v--)
                if ((v & 1) == odd && v * v <= 16 * m) vals[nvals++] = v;
            walk(T, m, odd, vals, nvals, cnt, 0, 24, 16 * m);
        }
    }
    return T;
}

constexpr Table kTable = make_table();
static_assert(!kTable.overflow && kTable.n == kClasses, "the 48-bit union has 383 classes of at most 5 groups");

}  // namespace search_cx
}  // namespace llvq
