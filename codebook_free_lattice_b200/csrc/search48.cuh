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
// codewords of weight 0, 8, 12, 16, 24 for the even classes of that weight), builds its G1 / G3
// (even: C_on / C_off) columns in shared memory in a sequential pass over the 24 ranks, and the
// warp walks the classes of the chunk together: the class is uniform across the warp, so its
// record (column offsets, steps da_g, criterion coefficients) is one broadcast read of shared
// memory, and each lane reads only its own column (conflict-free: element c of lane l at
// [c][l]).  Classes are grouped by their number of magnitude groups, so that each group count
// runs a fully unrolled loop.  All arithmetic is fp64.  The CTA
// keeps the best (criterion, class ordinal, codeword), ties going to the lower class ordinal and
// then the lower codeword mask, and warp 0 writes the point.
#pragma once
#include <climits>
#include <cstdint>

#include "device_common.cuh"
#include "kernels.cuh"

namespace llvq {

constexpr int kSrGroups = 5;       // distinct nonzero magnitudes a 48-bit class can have
constexpr int kSrClasses = 384;    // 383 classes of the 48-bit union
constexpr int kSrWarps = 6;        // two CTAs per SM: 2 x (6 warps x 12.8 KB of columns + the class table)
constexpr int kSrThreads = kSrWarps * 32;
constexpr int kSrEvenWeights = 5;  // even codeword weights 0, 8, 12, 16, 24
constexpr int kSrBlocks = 1 + kSrEvenWeights;   // class blocks: odd, then even by weight
constexpr int kSrCols = 25;        // entries of one set's column: counts 0..24
constexpr int kSrRowBytes = 32 * 8;             // one column entry for the warp's 32 lanes
constexpr int kSrOddChunks = 4096 / 32;

// One class as the kernel reads it (80 bytes, shared memory, the same class on every lane).
struct SearchRec48 {
    uint16_t off[kSrGroups];       // byte offset of the group's column entry: (kind * 25 + hi_g) * 256
                                   // (odd: 1- then 3-mod-4 kind; even: on S then off S)
    uint16_t id;                   // ordinal in index order (ties)
    uint8_t q;                     // even: parity of the negative signs the class needs on S
    uint8_t m;                     // shell
    uint8_t ng;                    // groups
    uint8_t pad_;
    double da[kSrGroups];          // a_g - a_{g+1} within the group's kind
    double turn;                   // even: 2 x the smallest 2-mod-4 magnitude (sign-turn cost per unit weight)
    double alpha, beta;            // criterion = alpha V + beta, set per launch (-inf: class off)
};
static_assert(sizeof(SearchRec48) == 80, "one class in 80 bytes");

// The part every CTA copies into shared memory.  Blocks: b = 0 the odd classes, b = 1 + w the
// even classes of codeword weight index w (0, 8, 12, 16, 24); within a block, classes by group
// count descending, those with G groups in [ng_base[b][5 - G], ng_base[b][6 - G]).  Codeword
// chunks: [0, kSrOddChunks) the odd codewords, kSrOddChunks + [chunk_base[w], chunk_base[w + 1])
// the even codewords of weight index w, by-weight slots [word_base[w], word_base[w + 1]).
struct SearchHead48 {
    SearchRec48 rec[kSrClasses];
    int n_odd;
    int ng_base[kSrBlocks][kSrGroups + 1];
    int word_base[kSrEvenWeights + 1];
    int chunk_base[kSrEvenWeights + 1];
    int pad_[3];
};
static_assert(sizeof(SearchHead48) % 16 == 0, "copied in 16-byte units");

// Device image: the head, then per class its group magnitudes (the point's reconstruction, read
// from global memory), then the codewords: [0, 4096) ascending mask (the odd classes' T),
// [4096, 8192) ascending (weight, mask) (the even classes' S).
constexpr int kSrWords = 8192;
struct SearchImage48 {
    SearchHead48 head;
    uint8_t mag[kSrClasses][8];
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
};

struct SearchSmem48 {
    SearchHead48 head;
    double col[kSrWarps][2 * kSrCols][32];        // per warp: entry e of lane l at [e][l]
    double w[24];                                 // |y| by rank (descending)
    int ord[24];                                  // rank -> position
    uint32_t pos;                                 // bit t: y >= 0 at rank t
    uint32_t negmask;                             // bit i: y_i < 0
    int bad;                                      // the row holds a NaN or an infinity
    int pad_;
    double red_f[kSrWarps];
    int red_j[kSrWarps], red_id[kSrWarps];
    uint32_t red_w[kSrWarps];
};
// two CTAs per SM: 228 KB per SM, 1 KB reserved per CTA
static_assert(2 * (sizeof(SearchSmem48) + 1024) <= 228 * 1024, "two CTAs per SM");

__device__ __forceinline__ bool sr_better(double f, int id, uint32_t w, double bf, int bid, uint32_t bw) {
    return f > bf || (f == bf && (id < bid || (id == bid && w < bw)));
}

__device__ __forceinline__ void sr_reduce(double &bf, int &bj, int &bid, uint32_t &bw) {
    for (int off = 16; off; off >>= 1) {
        const double of = __shfl_xor_sync(0xFFFFFFFFu, bf, off);
        const int oj = __shfl_xor_sync(0xFFFFFFFFu, bj, off), oid = __shfl_xor_sync(0xFFFFFFFFu, bid, off);
        const uint32_t ow = __shfl_xor_sync(0xFFFFFFFFu, bw, off);
        if (sr_better(of, oid, ow, bf, bid, bw)) { bf = of; bj = oj; bid = oid; bw = ow; }
    }
}

// the magnitude at descending rank r (0-based) among a class's magnitudes of one kind (0 past them)
__device__ __forceinline__ int sr_mag(const SearchRec48 &K, const uint8_t *mag, int second_kind, int r) {
    for (int g = 0; g < K.ng; g++) {
        const int e = K.off[g] / kSrRowBytes, kind = e >= kSrCols;
        if (kind == second_kind && r < e - kind * kSrCols) return mag[g];
    }
    return 0;
}

struct SrBest {
    double f;
    int j, id;
    uint32_t w;
};

// classes [jb, je) with G groups each, against this lane's column (colb: its entry 0)
template <bool ODD, int G>
__device__ __forceinline__ void sr_eval(const SearchRec48 *R, int jb, int je, const char *colb, uint32_t word,
                                        bool valid, int turn, double wlast, SrBest &b) {
#pragma unroll 2
    for (int j = jb; j < je; j++) {
        const SearchRec48 &K = R[j];
        double V = 0.0;
#pragma unroll
        for (int g = 0; g < G; g++) V = fma(K.da[g], *reinterpret_cast<const double *>(colb + K.off[g]), V);
        if (!ODD && turn != K.q) V = fma(-K.turn, wlast, V);
        const double f = fma(K.alpha, V, K.beta);
        if (valid && sr_better(f, K.id, word, b.f, b.id, b.w)) { b.f = f; b.j = j; b.id = K.id; b.w = word; }
    }
}

template <bool ODD>
__device__ __forceinline__ void sr_eval_block(const SearchRec48 *R, const int *nb, const char *colb, uint32_t word,
                                              bool valid, int turn, double wlast, SrBest &b) {
    sr_eval<ODD, 5>(R, nb[0], nb[1], colb, word, valid, turn, wlast, b);
    sr_eval<ODD, 4>(R, nb[1], nb[2], colb, word, valid, turn, wlast, b);
    sr_eval<ODD, 3>(R, nb[2], nb[3], colb, word, valid, turn, wlast, b);
    sr_eval<ODD, 2>(R, nb[3], nb[4], colb, word, valid, turn, wlast, b);
    sr_eval<ODD, 1>(R, nb[4], nb[5], colb, word, valid, turn, wlast, b);
}

__global__ void __launch_bounds__(kSrThreads, 2) k_search48(const SearchArgs48 a) {
    extern __shared__ __align__(16) unsigned char sr_raw[];
    SearchSmem48 &S = *reinterpret_cast<SearchSmem48 *>(sr_raw);
    const unsigned FULL = 0xFFFFFFFFu;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    load_smem_image(&S.head, &a.image->head, sizeof(SearchHead48));
    __syncthreads();
    for (int j = tid; j < kSrClasses; j += kSrThreads) {
        SearchRec48 &K = S.head.rec[j];
        const int m = K.m;
        const bool on = m >= 2 && m <= a.max_shell;
        const double al = a.mode == 0 ? 1.0 / sqrt(16.0 * (double)(m ? m : 1)) : 2.0 * a.scale;
        const double be = a.mode == 0 ? 0.0 : -a.scale * a.scale * 16.0 * (double)m;
        K.alpha = on ? al : 0.0;
        K.beta = on ? be : -INFINITY;
    }
    double(*col)[32] = S.col[warp];
    col[0][lane] = 0.0;                     // count 0 of either set: never rewritten
    col[kSrCols][lane] = 0.0;
    const char *colb = reinterpret_cast<const char *>(&col[0][lane]);
    const SearchRec48 *R = S.head.rec;
    const int n_odd = S.head.n_odd;
    const int n_chunks = kSrOddChunks + S.head.chunk_base[kSrEvenWeights];
    const bool act = lane < 24;
    __syncthreads();

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

        SrBest best{-INFINITY, -1, INT_MAX, 0u};
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
                while (e >= S.head.chunk_base[wi + 1]) wi++;
                const int t = S.head.word_base[wi] + (e - S.head.chunk_base[wi]) * 32 + lane;
                valid = t < S.head.word_base[wi + 1];
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
            if (odd) {                                      // continue each set past its end
                const double d = s1 - s2;
                for (int c = 1; c < kSrCols; c++) {
                    if (c > c1) col[c][lane] = d + col[kSrCols + 24 - c][lane];
                    if (c > c2) col[kSrCols + c][lane] = col[24 - c][lane] - d;
                }
                sr_eval_block<true>(R, S.head.ng_base[0], colb, word, true, 0, 0.0, best);
            } else {
                const int turn = __popc(word & negmask) & 1;
                sr_eval_block<false>(R, S.head.ng_base[1 + wi], colb, word, valid, turn, wlast, best);
            }
        }

        // ---- the best over the CTA -----------------------------------------------------------
        double bf = best.f;
        int bj = best.j, bid = best.id;
        uint32_t bw = best.w;
        sr_reduce(bf, bj, bid, bw);
        if (lane == 0) { S.red_f[warp] = bf; S.red_j[warp] = bj; S.red_id[warp] = bid; S.red_w[warp] = bw; }
        __syncthreads();
        if (warp == 0) {
            const int r = lane < kSrWarps ? lane : 0;
            bf = S.red_f[r]; bj = S.red_j[r]; bid = S.red_id[r]; bw = S.red_w[r];
            sr_reduce(bf, bj, bid, bw);
            // ---- the point of class bj and codeword bw (lane = rank) ---------------------
            const int j = bj < 0 ? 0 : bj;
            const SearchRec48 &K = R[j];
            const uint8_t *mag = a.image->mag[j];
            const int ord = act ? S.ord[lane] : 0;
            const double wt = act ? S.w[lane] : 0.0;
            const bool pos = (posb >> lane) & 1u;
            const unsigned le = lane == 31 ? FULL : (2u << lane) - 1u;
            const bool inw = (bw >> ord) & 1u;
            int x;
            if (j < n_odd) {
                const bool b = act && (inw == pos);
                const unsigned m1 = __ballot_sync(FULL, b);
                const int c1 = __popc(m1 & le), c3 = lane + 1 - c1;
                int n1 = 0;
                for (int g = 0; g < K.ng; g++) {
                    const int e = K.off[g] / kSrRowBytes;
                    if (e < kSrCols) n1 = max(n1, e);
                }
                const int n3 = 24 - n1;
                int mg;
                if (b) mg = c1 <= n1 ? sr_mag(K, mag, 0, c1 - 1) : sr_mag(K, mag, 1, n3 - 1 - (c1 - n1 - 1));
                else mg = c3 <= n3 ? sr_mag(K, mag, 1, c3 - 1) : sr_mag(K, mag, 0, n1 - 1 - (c3 - n3 - 1));
                x = (((mg & 3) == 1) == inw) ? mg : -mg;
            } else {
                const bool b = act && inw;
                const unsigned mS = __ballot_sync(FULL, b);
                const int con = __popc(mS & le), coff = lane + 1 - con;
                const int mg = b ? sr_mag(K, mag, 0, con - 1) : sr_mag(K, mag, 1, coff - 1);
                x = pos ? mg : -mg;
                const int turn = __popc(bw & negmask) & 1;
                if (mS && turn != K.q && lane == 31 - __clz(mS)) x = -x;
            }
            if (!act || bj < 0) x = 0;
            double d = (pos ? wt : -wt) * (double)x;
            for (int off = 16; off; off >>= 1) d += __shfl_xor_sync(FULL, d, off);
            if (act) a.points[v * 24 + ord] = (int8_t)x;
            if (lane == 0 && a.dots) a.dots[v] = d;
            if (a.codes) {                                   // nearest gain level to <y, v> / |v|
                const double g = d / sqrt(16.0 * (double)(K.m ? K.m : 1));
                double be = INFINITY;
                int bc = INT_MAX;
                for (int c = lane; c < a.n_levels; c += 32) {
                    const double e = fabs(g - a.levels[c]);
                    if (e < be) { be = e; bc = c; }
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
