// search48.cuh -- nearest point of the shell union Shell(2) u ... u Shell(M) of the 48-bit
// budget (M <= 13) to 24-dim inputs, by the angular or the Euclidean criterion; one CTA per
// input vector.
//
// "Leech Lattice Vector Quantization for Efficient LLM Compression": papernotes.org notes,
// 方法详解 / 关键设计 1 (multi-shell spherical and angular search over the union of shells;
// for the shape of a shape-gain split, input and candidates are unit vectors compared by their
// inner product) and gist.science, Methodik 2 (two criteria over the union: Euclidean distance
// for spherical shaping, cosine similarity for shape-gain; an extension of Adoul & Barth's
// single-shell search).
//
// Criteria, in sqrt(8)-scaled lattice coordinates (|v|^2 = 16 m on shell m):
//   angular   : maximize <y, v> / |v|;
//   Euclidean : maximize 2 c <y, v> - c^2 |v|^2, i.e. the nearest c v to y for a scale c > 0.
// All points of a class (magnitude multiset + coset) share one norm, so the search needs the
// largest <y, v> in each class.  For one Golay codeword that maximum is a closed form in prefix
// sums of the weights |y_i| sorted in descending order (the rearrangement inequality):
//   even class, codeword S (its 2-mod-4 positions): the 2-mod-4 magnitudes go to S and the
//     0-mod-4 ones elsewhere, each in descending order of |y_i|, signs those of y.  The sum
//     must be 0 mod 8, which fixes the parity of the negative signs on S; when y gives the
//     other parity, the smallest |y_i| on S (holding the smallest 2-mod-4 magnitude) turns:
//       V = sum_g da_g C_side(g)[hi_g] - turn * 2 a_min w_min.
//   odd class, codeword T (its 1-mod-4 positions): signs follow from T and the magnitudes, so
//     position i wants a 1-mod-4 magnitude when (i in T) equals (y_i >= 0).  With P1 / P3 the
//     two sets (sizes p1 + p3 = 24), C1 / C3 the prefix sums of the sorted weights in each
//     (totals t1, t3), the greedy assignment -- each set takes its own kind in descending order,
//     and a set with more positions than magnitudes of its kind gives its smallest weights the
//     other kind's smallest magnitudes with the wrong sign, the largest of those weights taking
//     the smallest magnitude -- is worth
//       V = sum_{1-mod-4 groups} da_g G1[hi_g] + sum_{3-mod-4 groups} da_g G3[hi_g],
//       G1[c] = C1[c] (c <= p1),  t1 - t3 + C3[24 - c] (c > p1),
//       G3[c] = C3[c] (c <= p3),  t3 - t1 + C1[24 - c] (c > p3)
//     (the Abel sum of the greedy value; the terms in t3 and t1 that carry each kind's largest
//     magnitude cancel because the da_g of a kind sum to that magnitude).
// da_g = a_g - a_{g+1} over one kind's distinct magnitudes in descending order (0 past the last),
// hi_g = how many of that kind's magnitudes are >= a_g.
//
// Work split: one CTA per input vector.  Warp 0 sorts the input into shared memory; then each
// lane owns one codeword (chunks of 32 codewords: the 4096 for the odd classes, then the even
// codewords of weight 0, 8, 12, 16, 24 for the even classes of that weight) and builds the prefix
// sums of its two sets in a sequential pass over the 24 ranks (a shared-memory column, element c
// of lane l at [c][l], conflict-free), loads the 50 entries into registers and, for odd
// codewords, continues each set past its end there.  The 383 classes of the union are a
// compile-time table (search48_classes.cuh, checked against the codec's class list when a codec
// is created), so every class is a straight-line chain of fp64 FMAs on registers with constant
// steps, four classes at a time (four independent chains, then one comparison with the running
// best).  A class list is in shell order, so a union short of shell 13 is a prefix of each list:
// those launches skip the quads past it, and the full union runs without any check.  The
// criterion is a template parameter: angular V / sqrt(16 m), Euclidean (divided by
// 2 c > 0, which keeps the order) V - 8 c m, with m and 1 / sqrt(16 m) compile-time constants.  The CTA
// keeps the best (criterion, class ordinal, codeword), ties going to the lower class ordinal and
// then the lower codeword mask, and warp 0 writes the point.
#pragma once
#include <climits>
#include <cstdint>
#include <utility>

#include "device_common.cuh"
#include "kernels.cuh"
#include "search48_classes.cuh"

namespace llvq {

constexpr int kSrGroups = search_cx::kGroups;
constexpr int kSrClasses = 384;    // 383 classes of the 48-bit union
constexpr int kSrWarps = 12;       // one CTA per SM: 12 x 12.8 KB of columns, about 168 registers a thread
constexpr int kSrThreads = kSrWarps * 32;
constexpr int kSrEvenWeights = 5;  // even codeword weights 0, 8, 12, 16, 24
constexpr int kSrCols = search_cx::kCols;
constexpr int kSrOddChunks = 4096 / 32;
constexpr int kSrWords = 8192;

// One class for the point's reconstruction (global memory, indexed by the class ordinal).
struct SearchRec48 {
    uint8_t e[kSrGroups];          // column entry: kind * 25 + count of the kind's magnitudes >= a_g
    uint8_t mag[kSrGroups];        // a_g
    uint8_t ng;                    // groups
    uint8_t m;                     // shell
    uint8_t odd;
    uint8_t q;                     // even: parity of the negative signs the class needs on S
    uint8_t pad_[2];
};
static_assert(sizeof(SearchRec48) == 16, "one class in 16 bytes");

// Device image: the class records by ordinal, the codeword chunk bounds and the codewords:
// [0, 4096) ascending mask (the odd classes' T), [4096, 8192) ascending (weight, mask) (the even
// classes' S).  Chunks: [0, kSrOddChunks) the odd codewords, kSrOddChunks + [chunk_base[w],
// chunk_base[w + 1]) the even codewords of weight index w, by-weight slots [word_base[w],
// word_base[w + 1]).
struct SearchImage48 {
    SearchRec48 rec[kSrClasses];
    int word_base[kSrEvenWeights + 1];
    int chunk_base[kSrEvenWeights + 1];
    uint32_t words[kSrWords];
};

struct SearchArgs48 {
    const SearchImage48 *image;
    int max_shell;
    int mode;                 // 0 angular, 1 Euclidean
    double scale;             // Euclidean reconstruction scale c
    const float *X;           // [n][24]
    long long n;
    int8_t *points;           // [n][24]
    double *dots;             // [n] or null: <y, v>
    const double *levels;     // gain levels (angular), or null
    int n_levels;
    uint8_t *codes;           // [n] nearest level to <y, v> / |v|, or null
    unsigned *flags;
    int nal[kSrEvenWeights + 1];   // per class list (odd, even by weight): classes in shells 2..max_shell
};


struct SearchSmem48 {
    double col[kSrWarps][2 * kSrCols][32];        // per warp: entry e of lane l at [e][l]
    double w[24];                                 // |y| by rank (descending)
    int ord[24];                                  // rank -> position
    uint32_t pos;                                 // bit t: y >= 0 at rank t
    uint32_t negmask;                             // bit i: y_i < 0
    int bad;                                      // the row holds a NaN or an infinity
    int pad_;
    int word_base[kSrEvenWeights + 1];
    int chunk_base[kSrEvenWeights + 1];
    int nal[kSrEvenWeights + 1];                  // per class list: how many of its classes lie in shells 2..max_shell
    double red_f[kSrWarps];
    int red_id[kSrWarps];
    uint32_t red_w[kSrWarps];
};
static_assert(sizeof(SearchSmem48) + 1024 <= 228 * 1024, "one CTA per SM");

__device__ __forceinline__ bool sr_better(double f, int id, uint32_t w, double bf, int bid, uint32_t bw) {
    return f > bf || (f == bf && (id < bid || (id == bid && w < bw)));
}

__device__ __forceinline__ void sr_reduce(double &bf, int &bid, uint32_t &bw) {
    for (int off = 16; off; off >>= 1) {
        const double of = __shfl_xor_sync(0xFFFFFFFFu, bf, off);
        const int oid = __shfl_xor_sync(0xFFFFFFFFu, bid, off);
        const uint32_t ow = __shfl_xor_sync(0xFFFFFFFFu, bw, off);
        if (sr_better(of, oid, ow, bf, bid, bw)) { bf = of; bid = oid; bw = ow; }
    }
}

// the magnitude at descending rank r (0-based) among a class's magnitudes of one kind (0 past them)
__device__ __forceinline__ int sr_mag(const SearchRec48 &K, int second_kind, int r) {
    for (int g = 0; g < K.ng; g++) {
        const int kind = K.e[g] >= kSrCols;
        if (kind == second_kind && r < K.e[g] - kind * kSrCols) return K.mag[g];
    }
    return 0;
}

struct SrBest {
    double f;
    int id;
    uint32_t w;
};

// 1 / sqrt(x) for the compile-time criterion constants (Newton's iteration from 0.1, which lies
// below sqrt(3 / x) for every x = 16 m <= 208, so the iteration converges; 12 steps reach the
// fp64 rounding level)
constexpr double sr_rsqrt(double x) {
    double y = 0.1;
    for (int i = 0; i < 12; i++) y = y * (1.5 - 0.5 * x * y * y);
    return y;
}

struct SrCrit {
    double nc8;               // Euclidean: -8 c
};

// criterion value of class J of the compile-time table against this lane's column entries
template <int MODE, int J>
__device__ __forceinline__ double sr_class(const double (&c)[2 * kSrCols], const SrCrit &cr, int turn,
                                           double wlast) {
    constexpr search_cx::Cls K = search_cx::kTable.c[J];
    double V = 0.0;
#pragma unroll
    for (int g = 0; g < K.ng; g++) V = fma((double)K.da[g], c[K.e[g]], V);
    if constexpr (!K.odd && K.k > 0) {
        if (turn != K.q) V = fma(-(double)K.turn2, wlast, V);
    }
    double f;
    if constexpr (MODE == 0) {
        constexpr double r = sr_rsqrt(16.0 * K.m);
        f = V * r;
    } else {
        f = fma((double)K.m, cr.nc8, V);
    }
    return f;
}

// class lists: 0 the odd classes, 1 + w the even classes of codeword weight index w
constexpr int sr_list_n(int list) {
    return list == 0 ? search_cx::kTable.n_odd : search_cx::kTable.n_even[list - 1];
}
constexpr int sr_list_id(int list, int i) {
    return list == 0 ? search_cx::kTable.odd_ids[i] : search_cx::kTable.even_ids[list - 1][i];
}

// the prefix of each class list (lists are in shell order) that lies in shells 2..max_shell (host)
inline void search_list_prefixes(int max_shell, int (&nal)[kSrEvenWeights + 1]) {
    for (int l = 0; l <= kSrEvenWeights; l++) {
        int n = 0;
        while (n < sr_list_n(l) && search_cx::kTable.c[sr_list_id(l, n)].m <= max_shell) n++;
        nal[l] = n;
    }
}

// classes B, B + 1, ... of list LST (up to four, ascending ordinals): four independent chains, the
// best of them (the lower ordinal on equal values), then one comparison with the running best.
// A list is in shell order, so the shells of the union are its first nal classes.  CHECK (a union
// short of shell 13): a quad past them is skipped, and the one that straddles the end masks its
// classes beyond it; without CHECK the quads run straight through.
template <int MODE, bool CHECK, int LST, int B>
__device__ __forceinline__ void sr_quad(const double (&c)[2 * kSrCols], const SrCrit &cr, int nal, uint32_t word,
                                        bool valid, int turn, double wlast, SrBest &b) {
    if constexpr (CHECK) {
        if (B >= nal) return;
    }
    constexpr int N = sr_list_n(LST);
    constexpr int j0 = sr_list_id(LST, B);
    double f = sr_class<MODE, j0>(c, cr, turn, wlast);
    int id = j0;
    if constexpr (B + 1 < N) {
        constexpr int j1 = sr_list_id(LST, B + 1);
        constexpr int j2 = sr_list_id(LST, B + 2 < N ? B + 2 : B + 1);
        constexpr int j3 = sr_list_id(LST, B + 3 < N ? B + 3 : B + 1);
        double f1 = sr_class<MODE, j1>(c, cr, turn, wlast);
        double f2 = -INFINITY, f3 = -INFINITY;
        if constexpr (B + 2 < N) f2 = sr_class<MODE, j2>(c, cr, turn, wlast);
        if constexpr (B + 3 < N) f3 = sr_class<MODE, j3>(c, cr, turn, wlast);
        if constexpr (CHECK) {
            if (B + 3 >= nal) {                      // the list's end falls in this quad
                f3 = -INFINITY;
                if (B + 2 >= nal) f2 = -INFINITY;
                if (B + 1 >= nal) f1 = -INFINITY;
            }
        }
        int id2 = j2;
        if (f1 > f) { f = f1; id = j1; }
        if (f3 > f2) { f2 = f3; id2 = j3; }
        if (f2 > f) { f = f2; id = id2; }
    }
    if (valid && f >= b.f && sr_better(f, id, word, b.f, b.id, b.w)) { b.f = f; b.id = id; b.w = word; }
}

template <int MODE, bool CHECK, int LST, int... Q>
__device__ __forceinline__ void sr_list(std::integer_sequence<int, Q...>, const double (&c)[2 * kSrCols],
                                        const SrCrit &cr, int nal, uint32_t word, bool valid, int turn,
                                        double wlast, SrBest &b) {
    (sr_quad<MODE, CHECK, LST, 4 * Q>(c, cr, nal, word, valid, turn, wlast, b), ...);
}

template <int MODE, int LST>
__device__ __forceinline__ void sr_block(const double (&c)[2 * kSrCols], const SrCrit &cr, const int *nal,
                                         bool full, uint32_t word, bool valid, int turn, double wlast, SrBest &b) {
    constexpr auto q = std::make_integer_sequence<int, (sr_list_n(LST) + 3) / 4>{};
    if (full) sr_list<MODE, false, LST>(q, c, cr, nal[LST], word, valid, turn, wlast, b);
    else sr_list<MODE, true, LST>(q, c, cr, nal[LST], word, valid, turn, wlast, b);
}

template <int MODE>
__global__ void __launch_bounds__(kSrThreads, 1) k_search48(const SearchArgs48 a) {
    extern __shared__ __align__(16) unsigned char sr_raw[];
    SearchSmem48 &S = *reinterpret_cast<SearchSmem48 *>(sr_raw);
    const unsigned FULL = 0xFFFFFFFFu;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const SrCrit cr{-8.0 * a.scale};
    if (tid < kSrEvenWeights + 1) {
        S.word_base[tid] = a.image->word_base[tid];
        S.chunk_base[tid] = a.image->chunk_base[tid];
    }
    if (tid == 0) {
#pragma unroll
        for (int l = 0; l <= kSrEvenWeights; l++) S.nal[l] = a.nal[l];   // constant indices: no local copy
    }
    double(*col)[32] = S.col[warp];
    col[0][lane] = 0.0;                     // count 0 of either set: never rewritten
    col[kSrCols][lane] = 0.0;
    const bool act = lane < 24;
    __syncthreads();
    const int n_chunks = kSrOddChunks + S.chunk_base[kSrEvenWeights];
    const bool full = a.max_shell >= search_cx::kShells;      // every class in the union

    for (long long v = blockIdx.x; v < a.n; v += gridDim.x) {
        // ---- warp 0: the input sorted by |y_i| descending (equal values by position) ---------
        if (warp == 0) {
            const double yi = act ? (double)a.X[v * 24 + lane] : 0.0;
            const double ai = fabs(yi);
            int rank = 0;
            for (int j = 0; j < 24; j++) {
                const double aj = __shfl_sync(FULL, ai, j);
                rank += (aj > ai) || (aj == ai && j < lane);
            }
            const bool fin = __all_sync(FULL, !act || isfinite(yi));
            const unsigned pos = __reduce_or_sync(FULL, act && !(yi < 0.0) ? 1u << rank : 0u);
            const unsigned neg = __ballot_sync(FULL, act && yi < 0.0);
            if (act) { S.w[rank] = ai; S.ord[rank] = lane; }
            if (lane == 0) { S.pos = pos; S.negmask = neg; S.bad = !fin; }
        }
        __syncthreads();
        if (S.bad) {                                        // the same branch on every warp
            if (warp == 0) {
                if (act) a.points[v * 24 + lane] = 0;
                if (lane == 0) {
                    if (a.dots) a.dots[v] = __longlong_as_double(0x7FF8000000000000ll);
                    if (a.codes) a.codes[v] = 0;
                    atomicOr(a.flags, kFlagSearchInput);
                }
            }
            __syncthreads();
            continue;
        }
        const uint32_t posb = S.pos, negmask = S.negmask;

        SrBest best{-INFINITY, INT_MAX, 0u};
        for (int ch = warp; ch < n_chunks; ch += kSrWarps) {
            // ---- this lane's codeword --------------------------------------------------------
            const bool odd = ch < kSrOddChunks;
            int wi = 0;
            uint32_t word = 0;
            bool valid = true;
            if (odd) {
                word = __ldg(a.image->words + ch * 32 + lane);
            } else {
                const int e = ch - kSrOddChunks;
                while (e >= S.chunk_base[wi + 1]) wi++;
                const int t = S.word_base[wi] + (e - S.chunk_base[wi]) * 32 + lane;
                valid = t < S.word_base[wi + 1];
                word = valid ? __ldg(a.image->words + 4096 + t) : 0u;
            }
            // ---- prefix sums of the sorted weights in the two sets, one pass over the ranks ----
            double s1 = 0.0, s2 = 0.0, wlast = 0.0;
            int c1 = 0, c2 = 0;
            for (int t = 0; t < 24; t++) {
                const double wt = S.w[t];
                const uint32_t inw = (word >> S.ord[t]) & 1u;
                const bool b = odd ? inw == ((posb >> t) & 1u) : inw != 0u;   // first set
                if (b) { s1 += wt; c1++; col[c1][lane] = s1; wlast = wt; }
                else { s2 += wt; c2++; col[kSrCols + c2][lane] = s2; }
            }
            double c[2 * kSrCols];
#pragma unroll
            for (int e = 0; e < 2 * kSrCols; e++) c[e] = (e % kSrCols) ? col[e][lane] : 0.0;
            if (odd) {
                // continue each set past its end: entries c > c1 of the first set read raw entries
                // 24 - c < c2 of the second, and the other way round, so the order is free
                const double d = s1 - s2;
#pragma unroll
                for (int e = 1; e < kSrCols; e++) {
                    if (e > c1) c[e] = d + c[kSrCols + 24 - e];
                    if (e > c2) c[kSrCols + e] = c[24 - e] - d;
                }
                sr_block<MODE, 0>(c, cr, S.nal, full, word, true, 0, 0.0, best);
            } else {
                const int turn = __popc(word & negmask) & 1;
                switch (wi) {
                    case 0: sr_block<MODE, 1>(c, cr, S.nal, full, word, valid, turn, wlast, best); break;
                    case 1: sr_block<MODE, 2>(c, cr, S.nal, full, word, valid, turn, wlast, best); break;
                    case 2: sr_block<MODE, 3>(c, cr, S.nal, full, word, valid, turn, wlast, best); break;
                    case 3: sr_block<MODE, 4>(c, cr, S.nal, full, word, valid, turn, wlast, best); break;
                    default: sr_block<MODE, 5>(c, cr, S.nal, full, word, valid, turn, wlast, best); break;
                }
            }
        }

        // ---- the best over the CTA -----------------------------------------------------------
        double bf = best.f;
        int bid = best.id;
        uint32_t bw = best.w;
        sr_reduce(bf, bid, bw);
        if (lane == 0) { S.red_f[warp] = bf; S.red_id[warp] = bid; S.red_w[warp] = bw; }
        __syncthreads();
        if (warp == 0) {
            const int r = lane < kSrWarps ? lane : 0;
            bf = S.red_f[r]; bid = S.red_id[r]; bw = S.red_w[r];
            sr_reduce(bf, bid, bw);
            // ---- the point of class bid and codeword bw (lane = rank) --------------------
            const bool found = bid >= 0 && bid < search_cx::kClasses;
            const SearchRec48 K = a.image->rec[found ? bid : 0];
            const int ord = act ? S.ord[lane] : 0;
            const double wt = act ? S.w[lane] : 0.0;
            const bool pos = (posb >> lane) & 1u;
            const unsigned le = lane == 31 ? FULL : (2u << lane) - 1u;
            const bool inw = (bw >> ord) & 1u;
            int x;
            if (K.odd) {
                const bool b = act && (inw == pos);
                const unsigned m1 = __ballot_sync(FULL, b);
                const int c1 = __popc(m1 & le), c3 = lane + 1 - c1;
                int n1 = 0;
                for (int g = 0; g < K.ng; g++)
                    if (K.e[g] < kSrCols) n1 = max(n1, (int)K.e[g]);
                const int n3 = 24 - n1;
                int mg;
                if (b) mg = c1 <= n1 ? sr_mag(K, 0, c1 - 1) : sr_mag(K, 1, n3 - 1 - (c1 - n1 - 1));
                else mg = c3 <= n3 ? sr_mag(K, 1, c3 - 1) : sr_mag(K, 0, n1 - 1 - (c3 - n3 - 1));
                x = (((mg & 3) == 1) == inw) ? mg : -mg;
            } else {
                const bool b = act && inw;
                const unsigned mS = __ballot_sync(FULL, b);
                const int con = __popc(mS & le), coff = lane + 1 - con;
                const int mg = b ? sr_mag(K, 0, con - 1) : sr_mag(K, 1, coff - 1);
                x = pos ? mg : -mg;
                const int turn = __popc(bw & negmask) & 1;
                if (mS && turn != K.q && lane == 31 - __clz(mS)) x = -x;
            }
            if (!act || !found) x = 0;
            double d = (pos ? wt : -wt) * (double)x;
            for (int off = 16; off; off >>= 1) d += __shfl_xor_sync(FULL, d, off);
            if (act) a.points[v * 24 + ord] = (int8_t)x;
            if (lane == 0 && a.dots) a.dots[v] = d;
            if (a.codes) {                                   // nearest gain level to <y, v> / |v|
                const double g = d / sqrt(16.0 * (double)(K.m ? K.m : 1));
                double be = INFINITY;
                int bc = INT_MAX;
                for (int cc = lane; cc < a.n_levels; cc += 32) {
                    const double e = fabs(g - a.levels[cc]);
                    if (e < be) { be = e; bc = cc; }
                }
                for (int off = 16; off; off >>= 1) {
                    const double oe = __shfl_xor_sync(FULL, be, off);
                    const int oc = __shfl_xor_sync(FULL, bc, off);
                    if (oe < be || (oe == be && oc < bc)) { be = oe; bc = oc; }
                }
                if (lane == 0) a.codes[v] = (uint8_t)(bc == INT_MAX ? 0 : bc);
            }
        }
        __syncthreads();                                     // S.w / S.ord / red_* of this vector
    }
}

}  // namespace llvq
