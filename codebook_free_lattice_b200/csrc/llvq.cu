// llvq.cu -- host side of libllvq: decode-table images for the 48-, 72- and 96-bit index
// budgets, kernel launches, and the C ABI declared in include/llvq.h.  Kernels: kernels.cuh,
// kernels_bin48.cuh, kernels_tc48.cuh; decoders: codec48.cuh, codec72.cuh, codec96.cuh; encoders:
// encode48.cuh, encode72.cuh, encode96.cuh; host table construction: tables.cpp, tables96.cpp.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <string>
#include <thread>
#include <type_traits>
#include <utility>
#include <vector>

#include "../../include/llvq.h"
#include "kernels.cuh"
#include "kernels_bin48.cuh"
#include "kernels_gemv48.cuh"
#include "kernels_tc.cuh"
#include "kernels_tc48.cuh"
#include "codec96.cuh"
#include "encode48.cuh"
#include "encode72.cuh"
#include "encode96.cuh"
#include "search48.cuh"
#include "gptq48.cuh"
#include "tables.h"
#include "tables96.h"

using namespace llvq;

static_assert(kFlagIndexRange == LLVQ_FLAG_INDEX_RANGE && kFlagWaitTimeout == LLVQ_FLAG_WAIT_TIMEOUT &&
                  kFlagNotCoded == LLVQ_FLAG_NOT_CODED && kFlagSearchInput == LLVQ_FLAG_SEARCH_INPUT,
              "device flag bits match the C ABI");

struct llvq_codec {
    int index_bits = 0;
    int device = -1;
    int M = 0;
    u128 npoints = 0;
    int64_t nclasses = 0;
    int num_sms = 0;
    void *d_image = nullptr;       // Smem48 / Smem72 image (copied to shared memory per CTA)
    Rec72 *d_recs72 = nullptr;     // 72-bit class records (global memory)
    uint32_t *d_guide72 = nullptr; // 72-bit guide table
    Rec96 *d_recs96 = nullptr;     // 96-bit class records (global memory)
    uint32_t *d_guide96 = nullptr; // 96-bit guide table (top 28 index bits)
    void *d_even48 = nullptr;      // SmemEven48 image (48-bit table path)
    uint32_t *d_tabC48 = nullptr;  // complement arrangement tables (48-bit table path)
    void *d_gv48 = nullptr;        // SmemGv48 image (48-bit fused products, k_gemv48)
    void *d_enc48 = nullptr;       // EncSmem48 image (48-bit encoder)
    void *d_search48 = nullptr;    // SearchImage48 (48-bit nearest-point search)
    void *d_enc72 = nullptr;       // EncSmem72 image (72-bit encoder)
    unsigned long long *d_keys72 = nullptr;  // 72-bit class keys (encoder)
    void *d_enc96 = nullptr;       // EncSmem96 image (96-bit encoder)
    unsigned long long *d_keys96 = nullptr;  // 96-bit class keys (encoder, built on the device)
    unsigned *d_flags = nullptr;   // sticky device flags
};

namespace {

thread_local std::string g_last_error;
// polls of a kernel's first bounded wait on its table copy and on its tensor-core products
// (llvq_set_wait_polls; tests set them to 0 to take the timeout paths)
std::atomic<uint32_t> g_first_wait_tries{kBulkWaitTries};
std::atomic<uint32_t> g_mma_wait_tries{kMmaWaitTries};

// 48-bit batches from this size up run on the tensor cores (k_gemm_tc48); smaller ones, and every
// 72/96-bit batch, on the CUDA cores
constexpr int kTensorCoreMinBatch = 8;
// 48-bit batch 1-2 products with at least this many blocks per SM run the warp-binned kernel
// (k_gemv48): 4-9% faster than the coset-sorted kernel on B200 from 11008x4104 up, slower on
// 4096x4104 (4.7k blocks per SM) and at batch 4
constexpr long long kWarpBinnedMinBlocks = 10000;

// smallest double >= n / d for small positive integers (directed rounding of the host division)
double round_up_ratio(double n, double d) {
    double r = n / d;
    while (std::fma(r, d, -n) < 0.0) r = std::nextafter(r, INFINITY);
    return r;
}


void fill_pdep(uint16_t off_tab[256], uint8_t tab[kPdepEntries]) {
    int off = 0;
    for (int mb = 0; mb < 256; mb++) {
        off_tab[mb] = (uint16_t)off;
        const int n = __builtin_popcount(mb);
        for (int bits = 0; bits < (1 << n); bits++) {
            uint32_t outb = 0;
            int src = 0;
            for (int pos = 0; pos < 8; pos++)
                if (mb >> pos & 1) { if (bits >> src & 1) outb |= 1u << pos; src++; }
            tab[off + bits] = (uint8_t)outb;
        }
        off += 1 << n;
    }
}

// per-group sign flag: odd coset -> |x| = 1 (mod 4); even coset -> |x| != 0
uint8_t sign_flag(const HostClass &c, int g) {
    const int v = c.vals[g];
    return (uint8_t)(c.odd ? (v % 4 == 1) : (v != 0));
}

// bytes g = 0..nbytes-1: cumulative counts C_<=g of the decode-order groups, saturating at 24
uint64_t cum_bytes(const HostClass &c, int nbytes) {
    uint64_t cum = 0;
    int acc = 0;
    for (int g = 0; g < nbytes; g++) {
        if (g < (int)c.cnts.size()) acc += c.cnts[g];
        cum |= (uint64_t)std::min(acc, 24) << (8 * g);
    }
    return cum;
}

llvq_status build_image48(const HostTables &T, Smem48 &S, std::string &err) {
    std::memset(&S, 0, sizeof S);
    if (T.classes.size() > 383 || T.M > 15) { err = "48-bit table larger than expected"; return LLVQ_ERR_UNSUPPORTED; }
    std::memcpy(S.golay_mask, T.golay_by_mask, sizeof S.golay_mask);
    std::memcpy(S.golay_weight, T.golay_by_weight, sizeof S.golay_weight);
    for (int c = 1; c < 32; c++) S.invc[c] = round_up_ratio(1.0, (double)c);
    const int nc = (int)T.classes.size();
    for (int i = 0; i < nc; i++) {
        const HostClass &c = T.classes[i];
        if (c.vals.size() > 5) { err = "more than 5 magnitude groups at 48 bits"; return LLVQ_ERR_UNSUPPORTED; }
        if (c.P >= ((u128)1 << 33) || c.P_C >= ((u128)1 << 24)) { err = "48-bit arrangement count out of range"; return LLVQ_ERR_UNSUPPORTED; }
        S.c_invP[i] = round_up_ratio(1.0, (double)c.P);    // P < 2^33: exact as a double
        S.c_invA[i] = round_up_ratio(1.0, (double)c.A);
        S.c_PC[i] = (double)c.P_C;                           // < 2^24 for every 48-bit class: exact
        uint32_t vals = 0, gflag = 0;
        for (int g = 0; g < 4 && g < (int)c.vals.size(); g++) {
            vals |= (uint32_t)c.vals[g] << (8 * g);
            gflag |= (uint32_t)sign_flag(c, g) << (8 * g);
        }
        S.c_cum[i] = (uint32_t)cum_bytes(c, 4);
        S.c_vals[i] = vals;
        S.c_gflag[i] = gflag;
        const uint32_t val4 = c.vals.size() > 4 ? (uint32_t)c.vals[4] : 0u;
        const uint32_t flag4 = c.vals.size() > 4 ? sign_flag(c, 4) : 0u;
        const uint32_t wbase = c.odd ? 0u : (uint32_t)T.weight_base[c.k];
        if (c.A > 0x1FFFu || c.B > 31 || c.m > 15 || val4 > 15 || wbase > 0xFFFu) {
            err = "48-bit class constant out of its field";
            return LLVQ_ERR_UNSUPPORTED;
        }
        S.c_info[i] = c.A | (uint32_t)c.B << 13 | (c.odd ? kInfoOdd : 0u) |
                      (((c.sum_abs / 4) & 1) ? kInfoParity : 0u) | (uint32_t)c.m << 21 | val4 << 25 | flag4 << 29;
        S.c_info2[i] = wbase | (uint32_t)(c.odd ? 24 : c.k) << 12;
        if (c.odd) {                                          // signed group values on / off T
            for (int g = 0; g < (int)c.vals.size(); g++) {
                const int a = c.vals[g];
                const unsigned long long on = (unsigned long long)(uint8_t)(int8_t)(a % 4 == 1 ? a : -a);
                const unsigned long long off = (unsigned long long)(uint8_t)(int8_t)(a % 4 == 3 ? a : -a);
                S.c_vt[i] |= on << (8 * g);
                S.c_vn[i] |= off << (8 * g);
            }
        }
        S.starts[i] = (unsigned long long)c.start;
    }
    S.starts[nc] = (unsigned long long)T.n_points;
    for (int i = nc + 1; i < 400; i++) S.starts[i] = ~0ull;
    // guide: bucket b -> class holding index b << shift (the last class past N_M)
    int lo = 0;
    for (int b = 0; b <= (1 << kGuideBits48); b++) {
        const unsigned long long first = (unsigned long long)b << kGuideShift48;
        while (lo + 1 < nc && S.starts[lo + 1] <= first) lo++;
        S.guide[b] = (uint16_t)lo;
    }
    fill_pdep(S.pdep_off, S.pdep);
    for (int m = 1; m < 16; m++) S.invnorm[m] = (float)(1.0 / (4.0 * std::sqrt((double)m)));
    return LLVQ_OK;
}

// Arrangement tables of the even-coset table path (see SmemEven48).  Classes whose codeword has
// weight 8, 12 or 16 and whose complement has at most kTabCMax arrangements are marked in their
// class info; every code sequence table is generated once per multiset of codes, in lexicographic
// order, by stepping through the distinct permutations.
constexpr uint64_t kTabCMax = 1u << 17;

uint32_t side_table(const std::vector<int> &codes_sorted, std::map<std::vector<int>, uint32_t> &index,
                    std::vector<uint32_t> &tab) {
    auto it = index.find(codes_sorted);
    if (it != index.end()) return it->second;
    const uint32_t off = (uint32_t)tab.size();
    std::vector<int> seq = codes_sorted;
    do {
        uint32_t e = 0;
        for (size_t i = 0; i < seq.size(); i++) e |= (uint32_t)seq[i] << (2 * i);
        tab.push_back(e);
    } while (std::next_permutation(seq.begin(), seq.end()));
    index[codes_sorted] = off;
    return off;
}

llvq_status build_even48(const HostTables &T, Smem48 &S, SmemEven48 &E, std::vector<uint32_t> &tabC,
                         std::string &err) {
    std::memset(&E, 0, sizeof E);
    std::map<std::vector<int>, uint32_t> idxS, idxC;
    std::vector<uint32_t> tabS;
    tabC.clear();
    for (size_t i = 0; i < T.classes.size(); i++) {
        const HostClass &c = T.classes[i];
        if (c.odd || (c.k != 8 && c.k != 12 && c.k != 16) || c.P_C > kTabCMax || c.P_S > 0x7FF) continue;
        std::vector<int> cs, cc;                   // value codes, ascending (groups are ascending)
        bool fits = true;
        for (size_t g = 0; g < c.vals.size(); g++) {
            const int v = c.vals[g];
            const int code = v % 4 == 2 ? (v - 2) / 4 : v / 4;
            if (code > 3) fits = false;
            for (int t = 0; t < c.cnts[g]; t++) (v % 4 == 2 ? cs : cc).push_back(code);
        }
        if (!fits) continue;
        const uint32_t offS = side_table(cs, idxS, tabS), offC = side_table(cc, idxC, tabC);
        if (offC > 0x7FFFFu || offS > 0x1FFFu || c.P_S > 0x7FFu) { err = "arrangement table offset out of its field"; return LLVQ_ERR_UNSUPPORTED; }
        S.c_offs[i] = offC | offS << 19;
        S.c_info2[i] |= (uint32_t)c.P_S << 17;
        S.c_info[i] |= kInfoTable;
        if (tabS.size() > (size_t)kTabS48) { err = "S arrangement table overflow"; return LLVQ_ERR_UNSUPPORTED; }
    }
    std::copy(tabS.begin(), tabS.end(), E.tabS);
    for (uint32_t mq = 0; mq < 16; mq++)
        for (uint32_t bits = 0; bits < 256; bits++) {
            const int n2 = 2 * __builtin_popcount(mq);
            uint32_t sb = bits & ((1u << n2) - 1u), cb = bits >> n2, e = 0;
            for (int pos = 0; pos < 4; pos++) {
                uint32_t mag, nz;
                if (mq >> pos & 1u) { mag = 2 + 4 * (sb & 3u); sb >>= 2; nz = 1; }
                else { mag = 4 * (cb & 3u); cb >>= 2; nz = mag != 0; }
                e |= mag << (8 * pos) | nz << (28 + pos);
            }
            E.merge[mq << 8 | bits] = e;
        }
    return LLVQ_OK;
}

// The image of the fused product kernel (SmemGv48), assembled from the decode image and the
// even-coset tables, plus the tables of the odd-coset fp16 path: the tail table of every multiset
// of 6 items over 4 groups, per-class cumulative counts and fp16 values on T, the pair sign masks
// of a nibble of negative flags, and the low codeword bits as a linear function of the top 12
// (checked against the whole code).
uint16_t fp16_bits(int v) {
    // exact for |v| <= 2048: sign, exponent, 10-bit mantissa
    if (v == 0) return 0;
    const uint16_t sign = v < 0 ? 0x8000 : 0;
    int a = v < 0 ? -v : v, e = 0;
    while ((a >> e) > 1) e++;
    const uint32_t mant = (uint32_t)((a << 10) >> e) & 0x3FFu;
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)mant);
}

llvq_status build_gv48(const HostTables &T, const Smem48 &S, const SmemEven48 &E, SmemGv48 &G, std::string &err) {
    std::memset(&G, 0, sizeof G);
    std::memcpy(G.starts, S.starts, sizeof G.starts);
    std::memcpy(G.c_invA, S.c_invA, sizeof G.c_invA);
    std::memcpy(G.c_invP, S.c_invP, sizeof G.c_invP);
    std::memcpy(G.c_PC, S.c_PC, sizeof G.c_PC);
    std::memcpy(G.invc, S.invc, sizeof G.invc);
    std::memcpy(G.c_info, S.c_info, sizeof G.c_info);
    std::memcpy(G.c_info2, S.c_info2, sizeof G.c_info2);
    std::memcpy(G.c_offs, S.c_offs, sizeof G.c_offs);
    std::memcpy(G.c_cum, S.c_cum, sizeof G.c_cum);
    std::memcpy(G.c_vals, S.c_vals, sizeof G.c_vals);
    std::memcpy(G.c_gflag, S.c_gflag, sizeof G.c_gflag);
    std::memcpy(G.invnorm, S.invnorm, sizeof G.invnorm);
    std::memcpy(G.tabS, E.tabS, sizeof G.tabS);
    std::memcpy(G.gweight, S.golay_weight, sizeof G.gweight);
    // even-coset fp16 merge: selectors (z, |x|/2) per coordinate, z = 8 on a nonzero coordinate
    for (uint32_t mq = 0; mq < 16; mq++)
        for (uint32_t bits = 0; bits < 256; bits++) {
            const int n2 = 2 * __builtin_popcount(mq);
            uint32_t sb = bits & ((1u << n2) - 1u), cb = bits >> n2, e = 0;
            for (int pos = 0; pos < 4; pos++) {
                uint32_t mag;
                if (mq >> pos & 1u) { mag = 2 + 4 * (sb & 3u); sb >>= 2; }
                else { mag = 4 * (cb & 3u); cb >>= 2; }
                const uint32_t sel = (mag != 0 ? 8u : 0u) | (mag / 2) << 4;   // nibbles z, |x|/2
                e |= sel << (8 * pos);
            }
            G.merge16[mq << 8 | bits] = e;
        }
    for (size_t i = 0; i < T.classes.size(); i++) {
        const HostClass &c = T.classes[i];
        if (c.odd || !(S.c_info[i] & kInfoTable)) continue;
        G.c_magS[i] = c.P_S == 1 ? 0u : (uint32_t)((((u128)1 << 32) + c.P_S - 1) / c.P_S);
    }
    std::memcpy(G.guide, S.guide, sizeof S.guide);
    std::memcpy(G.pdep_off, S.pdep_off, sizeof G.pdep_off);
    std::memcpy(G.pdep, S.pdep, sizeof S.pdep);
    // tail: multisets (n0, n1, n2, n3) of 6 items, arrangements lexicographic over groups 0 < 1 < 2 < 3
    uint32_t ntail = 0;
    for (int c0 = 0; c0 <= kOddTail48; c0++)
        for (int c1 = c0; c1 <= kOddTail48; c1++)
            for (int c2 = c1; c2 <= kOddTail48; c2++) {
                const int n[4] = {c0, c1 - c0, c2 - c1, kOddTail48 - c2};
                std::vector<int> seq;
                for (int g = 0; g < 4; g++)
                    for (int t = 0; t < n[g]; t++) seq.push_back(g);
                const uint32_t off = ntail;
                do {
                    uint32_t e = 0;
                    for (int k = 0; k < kOddTail48; k++) e |= (uint32_t)seq[k] << (2 * k);
                    if (ntail >= 4096) { err = "odd tail table overflow"; return LLVQ_ERR_UNSUPPORTED; }
                    G.tail[ntail++] = (uint16_t)e;
                } while (std::next_permutation(seq.begin(), seq.end()));
                G.tailc[c0 + 7 * c1 + 49 * c2] = make_uint2(off, ntail - off);
            }
    if (ntail != 4096) { err = "odd tail table size"; return LLVQ_ERR_UNSUPPORTED; }
    for (size_t i = 0; i < T.classes.size(); i++) {
        const HostClass &c = T.classes[i];
        if (!c.odd || c.vals.size() > 4) continue;
        G.c_cumodd[i] = (uint32_t)cum_bytes(c, 4) + 0x01010101u * (uint32_t)kOddBias48;
        uint32_t vt[2] = {0, 0};
        for (size_t g = 0; g < c.vals.size(); g++) {
            const int a = c.vals[g];
            const int on = a % 4 == 1 ? a : -a;        // x_i = a_i exactly when (i in T) == (a_i = 1 mod 4)
            vt[g / 2] |= (uint32_t)fp16_bits(on) << (16 * (g % 2));
        }
        G.c_vt[i][0] = vt[0];
        G.c_vt[i][1] = vt[1];
    }
    for (int nb = 0; nb < 16; nb++)                        // bit k: coordinate k of the nibble negative
        G.nsign[nb] = make_uint2(((nb & 1) ? 0x8000u : 0u) | ((nb & 2) ? 0x80000000u : 0u),
                                 ((nb & 4) ? 0x8000u : 0u) | ((nb & 8) ? 0x80000000u : 0u));
    for (int j = 0; j < 64; j++) {
        G.tlow[j] = (uint16_t)(T.golay_by_mask[j] & 0xFFFu);
        G.tlow[64 + j] = (uint16_t)(T.golay_by_mask[j << 6] & 0xFFFu);
    }
    for (uint32_t r = 0; r < 4096; r++) {
        const uint32_t w = r << 12 | (uint32_t)(G.tlow[r & 63u] ^ G.tlow[64u + (r >> 6)]);
        if (w != T.golay_by_mask[r]) { err = "Golay low bits are not linear in the top 12"; return LLVQ_ERR_UNSUPPORTED; }
    }
    return LLVQ_OK;
}

// Search tables of the 48-bit budget (k_search48).  The kernel's classes are a compile-time table
// (search48_classes.cuh); this checks it, class by class, against the codec's own list (shell,
// coset, magnitude multiset, and the column entries, steps and sign parity derived here from
// the HostClass), and writes what the point's reconstruction reads: per class its column entries
// and magnitudes, and the codewords by mask, then by (weight, mask).
llvq_status build_search48(const HostTables &T, SearchImage48 &I, std::string &err) {
    std::memset(&I, 0, sizeof I);
    static const int kWeights[kSrEvenWeights] = {0, 8, 12, 16, 24};
    const search_cx::Table &X = search_cx::kTable;
    if ((int)T.classes.size() != X.n || X.n > kSrClasses) { err = "search: class count differs from the compile-time table"; return LLVQ_ERR_UNSUPPORTED; }
    for (int id = 0; id < X.n; id++) {
        const HostClass &c = T.classes[id];
        const search_cx::Cls &x = X.c[id];
        // (magnitude, count) descending, zeros included, against the compile-time multiset
        std::vector<std::pair<int, int>> all;
        for (size_t g = 0; g < c.vals.size(); g++) all.push_back({c.vals[g], c.cnts[g]});
        std::sort(all.begin(), all.end(), [](auto a, auto b) { return a.first > b.first; });
        bool same = x.m == c.m && x.odd == (int)c.odd && x.nv == (int)all.size() && (c.odd || x.k == c.k);
        for (size_t g = 0; same && g < all.size(); g++) same = x.val[g] == all[g].first && x.cnt[g] == all[g].second;
        // groups of the two kinds, descending, with cumulative counts
        SearchRec48 &K = I.rec[id];
        int g = 0;
        for (int kd = 0; kd < 2 && same; kd++) {
            int cum = 0;
            std::vector<std::pair<int, int>> kind;
            for (auto &vc : all)
                if (vc.first != 0 && (c.odd ? (vc.first % 4 == 3) : (vc.first % 4 == 0)) == (kd == 1)) kind.push_back(vc);
            for (size_t u = 0; u < kind.size() && same; u++, g++) {
                if (g >= kSrGroups) { same = false; break; }
                cum += kind[u].second;
                const int next = u + 1 < kind.size() ? kind[u + 1].first : 0;
                K.e[g] = (uint8_t)(kd * kSrCols + cum);
                K.mag[g] = (uint8_t)kind[u].first;
                same = x.e[g] == K.e[g] && x.da[g] == kind[u].first - next;
            }
        }
        K.ng = (uint8_t)g;
        K.m = (uint8_t)c.m;
        K.odd = (uint8_t)c.odd;
        K.q = (uint8_t)(!c.odd && c.k > 0 ? (c.sum_abs / 4) & 1 : 0);
        same = same && x.ng == g && x.q == K.q;
        if (!same) { err = "search: compile-time class table differs from the codec's class " + std::to_string(id); return LLVQ_ERR_UNSUPPORTED; }
    }
    for (int w = 0; w < kSrEvenWeights; w++) I.word_base[w] = T.weight_base[kWeights[w]];
    I.word_base[kSrEvenWeights] = 4096;
    I.chunk_base[0] = 0;
    for (int w = 0; w < kSrEvenWeights; w++) {
        for (int t = I.word_base[w]; t < I.word_base[w + 1]; t++)
            if (__builtin_popcount(T.golay_by_weight[t]) != kWeights[w]) { err = "search: codeword weights"; return LLVQ_ERR_UNSUPPORTED; }
        I.chunk_base[w + 1] = I.chunk_base[w] + (I.word_base[w + 1] - I.word_base[w] + 31) / 32;
    }
    std::memcpy(I.words, T.golay_by_mask, 4096 * sizeof(uint32_t));
    std::memcpy(I.words + 4096, T.golay_by_weight, 4096 * sizeof(uint32_t));
    return LLVQ_OK;
}

// Encoder tables of the 48-bit budget: per class its count-vector key, digits and the groups of
// its two coordinate sets (set 0: off S, or all positions of an odd class; set 1: on S).
llvq_status build_enc48(const HostTables &T, EncSmem48 &E, std::string &err) {
    std::memset(&E, 0, sizeof E);
    std::memcpy(E.golay_mask, T.golay_by_mask, sizeof E.golay_mask);
    std::memcpy(E.golay_weight, T.golay_by_weight, sizeof E.golay_weight);
    for (int L = 2; L < 32; L++) E.mL[L] = (unsigned long long)((((u128)1 << 64) + L - 1) / L);
    for (int k = 0; k <= 24; k++) E.wbase[k] = (uint16_t)T.weight_base[k];
    // the top 12 coordinates must be an information set: codeword t of the mask order has top
    // bits t, so the encoder reads a codeword's place from its top 12 bits
    for (int t = 0; t < 4096; t++)
        if ((T.golay_by_mask[t] >> 12) != (uint32_t)t) { err = "Golay top 12 bits are not an information set"; return LLVQ_ERR_UNSUPPORTED; }
    for (int j = 0; j < 4096; j++) {
        const uint32_t w = T.golay_by_weight[j];
        E.wrank[w >> 12] = (uint16_t)(j - T.weight_base[__builtin_popcount(w)]);
    }
    const size_t nc = T.classes.size();
    if (nc > (size_t)kEncClasses48 || T.M >= kEncShells48) { err = "48-bit encoder table too small"; return LLVQ_ERR_UNSUPPORTED; }
    for (int m = 0; m < kEncShells48; m++)
        for (int o = 0; o < 2; o++) { E.seg_first[m][o] = 0; E.seg_count[m][o] = 0; }
    for (size_t i = 0; i < nc; i++) {
        const HostClass &c = T.classes[i];
        unsigned long long klo = 0;
        uint32_t khi = 0;
        for (size_t g = 0; g < c.vals.size(); g++) {
            const int v = c.vals[g];
            if (v > 13) { err = "48-bit class magnitude above 13"; return LLVQ_ERR_UNSUPPORTED; }
            if (v < 12) klo += (unsigned long long)c.cnts[g] << (5 * v);
            else khi += (uint32_t)c.cnts[g] << (5 * (v - 12));
        }
        E.key_lo[i] = klo;
        E.key_hi[i] = khi;
        E.info[i] = c.A | (uint32_t)c.B << 13 | (c.odd ? 1u : 0u) << 18 | (uint32_t)c.k << 19;
        E.start[i] = (unsigned long long)c.start;
        // set 1 = the codeword groups of an even class, set 0 = the rest (odd: every group)
        const int g1 = c.odd ? 0 : c.n_side0;
        const int first0 = c.odd ? 0 : c.n_side0, n0 = (int)c.vals.size() - first0;
        if (n0 > 8 || g1 > 4) { err = "48-bit class with too many groups for the encoder"; return LLVQ_ERR_UNSUPPORTED; }
        unsigned long long v0 = ~0ull, c0 = 0;
        uint32_t v1 = ~0u, c1 = 0;
        for (int g = 0; g < n0; g++) {
            v0 &= ~(0xFFull << (8 * g));
            v0 |= (unsigned long long)c.vals[first0 + g] << (8 * g);
            c0 |= (unsigned long long)c.cnts[first0 + g] << (8 * g);
        }
        for (int g = 0; g < g1; g++) {
            v1 &= ~(0xFFu << (8 * g));
            v1 |= (uint32_t)c.vals[g] << (8 * g);
            c1 |= (uint32_t)c.cnts[g] << (8 * g);
        }
        E.vals0[i] = v0;
        E.cnt0[i] = c0;
        E.vals1[i] = v1;
        E.cnt1[i] = c1;
        E.P0[i] = (unsigned long long)(c.odd ? c.P : c.P_C);
        E.P1[i] = (unsigned long long)(c.odd ? 1 : c.P_S);
        if (c.P > ((u128)1 << 40)) { err = "48-bit arrangement count above 2^40"; return LLVQ_ERR_UNSUPPORTED; }
        const int o = c.odd ? 1 : 0;
        if (E.seg_count[c.m][o] == 0) E.seg_first[c.m][o] = (uint16_t)i;
        E.seg_count[c.m][o]++;
        // classes of one shell and coset must ascend by key (the order the search relies on)
        if (E.seg_count[c.m][o] > 1 &&
            !(E.key_hi[i - 1] < khi || (E.key_hi[i - 1] == khi && E.key_lo[i - 1] < klo))) {
            err = "48-bit class keys out of order";
            return LLVQ_ERR_UNSUPPORTED;
        }
    }
    return LLVQ_OK;
}

// Encoder tables of the 72-bit budget: the unary class keys (one per class, index order), the
// (shell, coset) ranges, and the shared-memory image (Golay masks, ranks within weight, binomials).
llvq_status build_enc72(const HostTables &T, EncSmem72 &E, std::vector<unsigned long long> &keys, std::string &err) {
    std::memset(&E, 0, sizeof E);
    std::memcpy(E.golay_mask, T.golay_by_mask, sizeof E.golay_mask);
    for (int t = 0; t < 4096; t++)
        if ((T.golay_by_mask[t] >> 12) != (uint32_t)t) { err = "Golay top 12 bits are not an information set"; return LLVQ_ERR_UNSUPPORTED; }
    for (int j = 0; j < 4096; j++) {
        const uint32_t w = T.golay_by_weight[j];
        E.wrank[w >> 12] = (uint16_t)(j - T.weight_base[__builtin_popcount(w)]);
    }
    for (int L = 2; L < 32; L++) E.mL[L] = (unsigned long long)((((u128)1 << 64) + L - 1) / L);
    for (int n = 0; n <= 24; n++)
        for (int c = 0; c <= 24; c++) {
            u128 b = 0;
            if (c <= n) { b = 1; for (int i = 0; i < c; i++) b = b * (u128)(n - i) / (u128)(i + 1); }
            E.binom[n][c] = (uint32_t)b;
        }
    if (T.M >= kEncShells72) { err = "72-bit encoder segment table too small"; return LLVQ_ERR_UNSUPPORTED; }
    const size_t nc = T.classes.size();
    keys.assign(nc, 0);
    for (size_t i = 0; i < nc; i++) {
        const HostClass &c = T.classes[i];
        int cnt[15] = {0};
        for (size_t g = 0; g < c.vals.size(); g++) {
            if (c.vals[g] > 29) { err = "72-bit class magnitude above 29"; return LLVQ_ERR_UNSUPPORTED; }
            cnt[c.vals[g] >> 1] += c.cnts[g];
        }
        unsigned long long key = 0;
        for (int b = 14; b >= 0; b--) key = (key << (cnt[b] + 1)) | (((1ull << cnt[b]) - 1ull) << 1);
        keys[i] = key;
        if (c.P > ((u128)1 << 52)) { err = "72-bit arrangement count above 2^52"; return LLVQ_ERR_UNSUPPORTED; }
        const int o = c.odd ? 1 : 0;
        if (E.seg_count[c.m][o] == 0) E.seg_first[c.m][o] = (uint32_t)i;
        else if (keys[i - 1] >= key) { err = "72-bit class keys out of order"; return LLVQ_ERR_UNSUPPORTED; }
        E.seg_count[c.m][o]++;
    }
    return LLVQ_OK;
}

llvq_status build_image72(const HostTables &T, Smem72 &S, std::vector<Rec72> &recs,
                          std::vector<uint32_t> &guide, std::string &err) {
    std::memset(&S, 0, sizeof S);
    if (T.M > 63) { err = "72-bit table larger than expected"; return LLVQ_ERR_UNSUPPORTED; }
    std::memcpy(S.golay_mask, T.golay_by_mask, sizeof S.golay_mask);
    std::memcpy(S.golay_weight, T.golay_by_weight, sizeof S.golay_weight);
    for (int c = 2; c < 32; c++) S.rc[c] = (unsigned long long)((((u128)1 << 64) + c - 1) / c);
    const size_t nc = T.classes.size();
    recs.assign(nc + 1, Rec72{});
    for (size_t i = 0; i < nc; i++) {
        const HostClass &c = T.classes[i];
        if (c.vals.size() > 9) { err = "more than 9 magnitude groups at 72 bits"; return LLVQ_ERR_UNSUPPORTED; }
        // 24 * 577 * P <= 2^64 keeps every fixed-point slot exact (see codec72.cuh)
        if (c.P * (u128)(24 * 577) > ((u128)1 << 64)) { err = "arrangement count above the fixed-point bound"; return LLVQ_ERR_UNSUPPORTED; }
        Rec72 &R = recs[i];
        R.start_lo = (unsigned long long)c.start;
        R.start_hi = (unsigned long long)(c.start >> 64);
        if (c.P > 1) {
            const u128 two64 = (u128)1 << 64;
            R.Rint = (unsigned long long)(two64 / c.P);
            const u128 rem = two64 % c.P;               // fraction rem / P, times 2^64, rounded up
            R.Rfrac = (unsigned long long)(((rem << 64) + c.P - 1) / c.P);
        }
        R.PC = (unsigned long long)c.P_C;
        R.mA = ~0ull / c.A;
        R.cum = cum_bytes(c, 8);
        for (int g = 0; g < 8 && g < (int)c.vals.size(); g++) {
            R.vals |= (unsigned long long)c.vals[g] << (8 * g);
            if (g < 4) R.flo |= (uint32_t)sign_flag(c, g) << (8 * g);
            else R.fhi |= (uint32_t)sign_flag(c, g) << (8 * (g - 4));
        }
        R.val8 = c.vals.size() > 8 ? (uint8_t)c.vals[8] : 0;
        R.flag8 = c.vals.size() > 8 ? sign_flag(c, 8) : 0;
        R.A = c.A;
        R.nS = (uint8_t)(c.odd ? 24 : c.k);
        R.B = (uint8_t)c.B;
        R.flags = (uint8_t)((c.odd ? 1 : 0) | (((c.sum_abs / 4) & 1) << 1));
        R.m = (uint8_t)c.m;
        R.ngroups = (uint8_t)c.vals.size();
        R.wbase = (uint16_t)(c.odd ? 0 : T.weight_base[c.k]);
    }
    recs[nc].start_lo = (unsigned long long)T.n_points;        // sentinel
    recs[nc].start_hi = (unsigned long long)(T.n_points >> 64);
    guide.assign((1u << kGuideBits72) + 1, 0);
    size_t lo = 0;
    for (uint32_t b = 0; b <= (1u << kGuideBits72); b++) {
        const u128 first = (u128)b << (72 - kGuideBits72);
        while (lo + 1 < nc && T.classes[lo + 1].start <= first) lo++;
        guide[b] = (uint32_t)lo;
    }
    fill_pdep(S.pdep_off, S.pdep);
    for (int m = 1; m < 64; m++) S.invnorm[m] = (float)(1.0 / (4.0 * std::sqrt((double)m)));
    return LLVQ_OK;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

Dec48::Args args48(const llvq_codec *c) {
    return Dec48::Args{(const Smem48 *)c->d_image, (unsigned long long)c->npoints};
}
Dec72::Args args72(const llvq_codec *c) {
    return Dec72::Args{(const Smem72 *)c->d_image, c->d_recs72, c->d_guide72,
                       (unsigned long long)c->npoints, (unsigned long long)(c->npoints >> 64)};
}

Dec96::Args args96(const llvq_codec *c) {
    return Dec96::Args{(const Smem96 *)c->d_image, c->d_recs96, c->d_guide96, (unsigned long long)c->npoints,
                       (uint32_t)(c->npoints >> 64)};
}

// guide[b] = the class holding index b 2^68 (the last class whose start is <= b 2^68)
__global__ void k_guide96(const Rec96 *__restrict__ recs, long long ncls, uint32_t *__restrict__ guide, long long nb) {
    const long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= nb) return;
    const unsigned long long thi = (unsigned long long)b << (kGuideShift96 - 64);
    if (thi > 0xFFFFFFFFull) { guide[b] = (uint32_t)(ncls - 1); return; }
    long long lo = 0, hi = ncls - 1;
    while (lo < hi) {
        const long long mid = (lo + hi + 1) >> 1;
        const uint32_t sh = recs[mid].start_hi;
        const bool le = sh < (uint32_t)thi || (sh == (uint32_t)thi && recs[mid].start_lo == 0ull);
        if (le) lo = mid; else hi = mid - 1;
    }
    guide[b] = (uint32_t)lo;
}

// The 96-bit tables: shell sizes and class counts on the host, then the class records shell by
// shell on the host threads, each shell copied to its place in the device table, then the guide
// on the device.
llvq_status create96(llvq_codec *c, std::vector<unsigned char> &image, std::string &err) {
    Tables96 T;
    const int hw = std::max(1, (int)std::thread::hardware_concurrency());
    if (!build_tables96(T, hw, err)) return LLVQ_ERR_UNSUPPORTED;
    c->M = T.M;
    c->npoints = T.n_points;
    c->nclasses = T.n_classes;
    image.assign(sizeof(Smem96), 0);
    Smem96 &S = *reinterpret_cast<Smem96 *>(image.data());
    std::memcpy(S.golay_mask, T.golay_by_mask, sizeof S.golay_mask);
    std::memcpy(S.golay_weight, T.golay_by_weight, sizeof S.golay_weight);
    for (int d = 2; d < 32; d++) S.mc[d] = (unsigned long long)((((u128)1 << 64) + d - 1) / d);
    for (int k = 0; k <= 24; k++) {
        S.nwords[k] = (uint16_t)T.words_of_weight[k];
        S.wbase[k] = (uint16_t)T.weight_base[k];
        const int A = T.words_of_weight[k];
        if (A >= 2) S.mA[k] = (unsigned long long)((((u128)1 << 64) + A - 1) / A);
    }
    S.nwords[25] = 4096;
    S.mA[25] = 1ull << 52;
    for (int n = 1; n <= 24; n++) {             // directed roundings keep the log2 P_i bound above
        const double l = std::log2((double)n);
        float dn = (float)l, up = (float)l;
        while ((double)dn > l) dn = std::nextafter(dn, -INFINITY);
        while ((double)up < l) up = std::nextafter(up, INFINITY);
        S.lg2_down[n] = dn;
        S.lg2_up[n] = up;
    }
    fill_pdep(S.pdep_off, S.pdep);
    if (T.M > 255) { err = "96-bit shell bound above the table"; return LLVQ_ERR_UNSUPPORTED; }
    for (int m = 1; m <= T.M; m++) S.invnorm[m] = (float)(1.0 / (4.0 * std::sqrt((double)m)));
    const long long nb = (long long)((T.n_points - 1) >> kGuideShift96) + 2;
    if (cudaMalloc(&c->d_recs96, (size_t)T.n_classes * sizeof(Rec96)) != cudaSuccess ||
        cudaMalloc(&c->d_guide96, (size_t)nb * sizeof(uint32_t)) != cudaSuccess) {
        err = "device memory for the 96-bit class table (" +
              std::to_string((size_t)T.n_classes * sizeof(Rec96) + (size_t)nb * 4) + " bytes) not available";
        cudaGetLastError();
        return LLVQ_ERR_CUDA;
    }
    // fill threads hold one shell each (up to 0.6 GB of records)
    const int nfill = std::min(hw, 8);
    std::atomic<int> next(0);
    std::atomic<bool> failed(false);
    std::mutex emu;
    std::vector<std::thread> pool;
    for (int th = 0; th < nfill; th++)
        pool.emplace_back([&]() {
            if (cudaSetDevice(c->device) != cudaSuccess) { failed = true; return; }
            std::vector<Rec96> buf;
            std::string e;
            while (!failed) {
                const int m = T.M - next.fetch_add(1);
                if (m < 2) break;
                buf.resize((size_t)T.shell_classes[m]);
                if (!fill_shell96(T, m, buf.data(), e) ||
                    cudaMemcpy(c->d_recs96 + T.class_base[m], buf.data(), buf.size() * sizeof(Rec96),
                               cudaMemcpyHostToDevice) != cudaSuccess) {
                    std::lock_guard<std::mutex> g(emu);
                    if (!failed) err = e.empty() ? "copy of the 96-bit class records failed" : e;
                    failed = true;
                }
            }
        });
    for (auto &t : pool) t.join();
    if (failed) return LLVQ_ERR_UNSUPPORTED;
    k_guide96<<<(unsigned)((nb + 255) / 256), 256>>>(c->d_recs96, T.n_classes, c->d_guide96, nb);
    if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
        err = "96-bit guide construction failed";
        return LLVQ_ERR_CUDA;
    }
    // encoder: class keys on the device, (shell, coset) ranges and small tables in an image
    if (cudaMalloc(&c->d_keys96, (size_t)T.n_classes * sizeof(unsigned long long)) != cudaSuccess) {
        err = "device memory for the 96-bit class keys not available";
        cudaGetLastError();
        return LLVQ_ERR_CUDA;
    }
    k_keys96<<<(unsigned)((T.n_classes + 255) / 256), 256>>>(c->d_recs96, T.n_classes, c->d_keys96);
    if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
        err = "96-bit class keys failed";
        return LLVQ_ERR_CUDA;
    }
    std::vector<unsigned char> eimg(sizeof(EncSmem96), 0);
    EncSmem96 &E = *reinterpret_cast<EncSmem96 *>(eimg.data());
    std::memcpy(E.golay_mask, T.golay_by_mask, sizeof E.golay_mask);
    for (int t = 0; t < 4096; t++)
        if ((T.golay_by_mask[t] >> 12) != (uint32_t)t) { err = "Golay top 12 bits are not an information set"; return LLVQ_ERR_UNSUPPORTED; }
    for (int j = 0; j < 4096; j++) {
        const uint32_t w = T.golay_by_weight[j];
        E.wrank[w >> 12] = (uint16_t)(j - T.weight_base[__builtin_popcount(w)]);
    }
    for (int L = 2; L < 32; L++) E.mL[L] = (unsigned long long)((((u128)1 << 64) + L - 1) / L);
    for (int n = 0; n <= 24; n++)
        for (int k = 0; k <= 24; k++) {
            u128 b = 0;
            if (k <= n) { b = 1; for (int i = 0; i < k; i++) b = b * (u128)(n - i) / (u128)(i + 1); }
            E.binom[n][k] = (uint32_t)b;
        }
    for (int k = 0; k <= 24; k++) E.nwords[k] = (uint16_t)T.words_of_weight[k];
    if (T.M >= kEncShells96) { err = "96-bit encoder segment table too small"; return LLVQ_ERR_UNSUPPORTED; }
    for (int m = 2; m <= T.M; m++) {
        E.seg_first[m][0] = (uint32_t)T.class_base[m];
        E.seg_count[m][0] = (uint32_t)T.shell_even[m];
        E.seg_first[m][1] = (uint32_t)(T.class_base[m] + T.shell_even[m]);
        E.seg_count[m][1] = (uint32_t)(T.shell_classes[m] - T.shell_even[m]);
    }
    if (cudaMalloc(&c->d_enc96, eimg.size()) != cudaSuccess ||
        cudaMemcpy(c->d_enc96, eimg.data(), eimg.size(), cudaMemcpyHostToDevice) != cudaSuccess) {
        err = "device allocation for the 96-bit encoder failed";
        cudaGetLastError();
        return LLVQ_ERR_CUDA;
    }
    return LLVQ_OK;
}

template <class D>
cudaError_t launch_decode(const llvq_codec *c, typename D::Args a, const void *words, long long n,
                          int8_t *out, cudaStream_t st) {
    if constexpr (std::is_same<D, Dec48>::value) {
        // coset-sorted decode: one 1024-thread CTA per SM over a contiguous range of words
        if (n == 0) return cudaSuccess;
        const int grid = (int)std::max(1LL, std::min((long long)c->num_sms, (n + kBinThreads - 1) / kBinThreads));
        const long long per = (n + grid - 1) / grid;
        if (per >= (1LL << 31)) return cudaErrorInvalidValue;
        DecodeSink sink{};
        sink.words = (const unsigned long long *)words;
        sink.n = n;
        sink.out = out;
        sink.per_cta = per;
        k_bin48<DecodeSink, kBinPer><<<grid, kBinThreads, bin48_base_smem(kBinPer), st>>>(
            a, (const SmemEven48 *)c->d_even48, c->d_tabC48, sink, c->d_flags, g_first_wait_tries.load());
        return cudaGetLastError();
    }
    const int threads = 512;
    const long long want = (n + threads - 1) / threads;
    const int grid = (int)std::max(1LL, std::min(want, (long long)c->num_sms * D::kCtasPerSm));
    k_decode<D><<<grid, threads, sizeof(typename D::Smem), st>>>(a, (const typename D::Word *)words, n, out,
                                                                c->d_flags);
    return cudaGetLastError();
}

template <class D, int B>
cudaError_t launch_gemm(const llvq_codec *c, typename D::Args a, const llvq_weight *w, const void *X,
                        float *Y, cudaStream_t st, int batch = B) {
    const int threads = 512;
    int grid = c->num_sms * gemm_ctas_per_sm<D, B>();
    int rpc = std::max((w->rows + grid - 1) / grid, 1);
    grid = (w->rows + rpc - 1) / rpc;
    const size_t smem = sizeof(typename D::Smem) + (size_t)B * rpc * gemm_acc_slots<B>() * sizeof(float);
    const int nb = w->blocks_per_row;
    // block index -> row by a multiply-high: exact while rpc * nb < 2^32 / nb
    if ((unsigned long long)rpc * nb * nb >= (1ull << 32)) return cudaErrorInvalidValue;
    if (smem > 200 * 1024) return cudaErrorInvalidValue;
    const uint32_t recip = nb > 1 ? (uint32_t)(((1ull << 32) + nb - 1) / nb) : 0u;
    k_gemm<D, B><<<grid, threads, smem, st>>>(a, (const typename D::Word *)w->words, w->row_pitch_words,
                                             w->rows, nb, recip, w->gain_mode, (const __half *)w->gains,
                                             (const __half *)X, Y, rpc, batch, c->d_flags);
    return cudaGetLastError();
}

template <class D, int... Bs>
void set_gemm_attrs(std::integer_sequence<int, Bs...>) {
    (cudaFuncSetAttribute(k_gemm<D, Bs + 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024), ...);
    cudaFuncSetAttribute(k_gemm<D, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    cudaFuncSetAttribute(k_gemm<D, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
}

constexpr size_t kBinSmemLimit = 232448;          // opt-in shared memory per block on sm_100

template <int... Bs>
void set_bin48_attrs(std::integer_sequence<int, Bs...>) {
    (cudaFuncSetAttribute(k_bin48<GemvSink<Bs + 1>, 5>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                          (int)kBinSmemLimit), ...);
    (cudaFuncSetAttribute(k_bin48<GemvSink<Bs + 1>, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                          (int)kBinSmemLimit), ...);
    cudaFuncSetAttribute(k_bin48<DecodeSink, kBinPer>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)kBinSmemLimit);
}

// The coset-sorted product (k_bin48 with GemvSink): one CTA per SM over a row range, the whole
// range classified in chunks of up to 5 blocks per thread.
template <int B>
cudaError_t launch_gemm_bin48(const llvq_codec *c, Dec48::Args a, const llvq_weight *w, const void *X, float *Y,
                              cudaStream_t st) {
    const int nb = w->blocks_per_row;
    if (nb > 0xFFFF) return cudaErrorInvalidValue;                  // column field of a record
    // one CTA per SM over a row range; 5 blocks per thread and chunk when the row accumulators
    // leave room, else 4, else the row range shrinks (more CTAs than SMs)
    int rpc = std::max(1, (w->rows + c->num_sms - 1) / c->num_sms);
    int per = bin48_smem_bytes(B, rpc, 5) <= kBinSmemLimit ? 5 : 4;
    while (rpc > 1 && bin48_smem_bytes(B, rpc, per) > kBinSmemLimit) rpc = (rpc + 1) / 2;
    if (bin48_smem_bytes(B, rpc, per) > kBinSmemLimit) return cudaErrorInvalidValue;
    // block index -> row by a multiply-high: exact while rpc * nb < 2^32 / nb
    if ((unsigned long long)rpc * nb * nb >= (1ull << 32)) return cudaErrorInvalidValue;
    const int grid = (w->rows + rpc - 1) / rpc;
    const uint32_t recip = nb > 1 ? (uint32_t)(((1ull << 32) + nb - 1) / nb) : 0u;
    GemvSink<B> sink{};
    sink.words = (const unsigned long long *)w->words;
    sink.pitch = w->row_pitch_words;
    sink.rows = w->rows;
    sink.nb = nb;
    sink.nb_recip = recip;
    sink.gain_mode = w->gain_mode;
    sink.gains = (const __half *)w->gains;
    sink.X = (const __half *)X;
    sink.Y = Y;
    sink.rows_per_cta = rpc;
    auto kern = per == 5 ? k_bin48<GemvSink<B>, 5> : k_bin48<GemvSink<B>, 4>;
    kern<<<grid, kBinThreads, bin48_smem_bytes(B, rpc, per), st>>>(a, (const SmemEven48 *)c->d_even48,
                                                                  c->d_tabC48, sink, c->d_flags,
                                                                  g_first_wait_tries.load());
    return cudaGetLastError();
}

// 48-bit products of batch 1..7 (k_gemv48): one CTA per SM over a row range; the row range
// shrinks (more CTAs than SMs) when the row accumulators would not fit next to the tables.
template <int B>
cudaError_t launch_gemv48(const llvq_codec *c, Dec48::Args a, const llvq_weight *w, const void *X, float *Y,
                          cudaStream_t st) {
    const int nb = w->blocks_per_row;
    if (nb > 0xFFFF) return cudaErrorInvalidValue;                  // column field of a record
    const int rpc = std::max(1, (w->rows + c->num_sms - 1) / c->num_sms);
    if (rpc > 0xFFFF) return cudaErrorInvalidValue;                 // row field of a record
    // block index -> row by a multiply-high: exact while rpc * nb < 2^32 / nb
    if ((unsigned long long)rpc * nb * nb >= (1ull << 32)) return cudaErrorInvalidValue;
    const size_t smem = gv48_smem_bytes(B, nb, false);   // activations read through L1
    GvArgs g{};
    g.image = (const SmemGv48 *)c->d_gv48;
    g.npoints = a.npoints;
    g.tabC = c->d_tabC48;
    g.words = (const unsigned long long *)w->words;
    g.pitch = w->row_pitch_words;
    g.rows = w->rows;
    g.nb = nb;
    g.nb_recip = nb > 1 ? (uint32_t)(((1ull << 32) + nb - 1) / nb) : 0u;
    g.gain_mode = w->gain_mode;
    g.gains = (const __half *)w->gains;
    g.X = (const __half *)X;
    g.Y = Y;
    g.rows_per_cta = rpc;
    g.wait_tries = g_first_wait_tries.load();
    // programmatic dependent launch: this kernel's table copy may overlap the end of the previous
    // kernel on the stream (the kernel waits for it before touching any data)
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((w->rows + rpc - 1) / rpc));
    cfg.blockDim = dim3(kGvThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    unsigned *flags = c->d_flags;
    const bool direct = w->gain_mode == LLVQ_GAIN_FP16_DIRECT;
    if (direct) return cudaLaunchKernelEx(&cfg, k_gemv48<B, 0, false>, g, flags);
    return cudaLaunchKernelEx(&cfg, k_gemv48<B, 1, false>, g, flags);
}

template <int... Bs>
void set_gemv48_attrs(std::integer_sequence<int, Bs...>) {


    (cudaFuncSetAttribute(k_gemv48<Bs + 1, 0, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBinSmemLimit), ...);
    (cudaFuncSetAttribute(k_gemv48<Bs + 1, 1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBinSmemLimit), ...);

}

// 48-bit tensor-core path: 128-row tiles x K splits of 8-block rounds.  The split is chosen to
// minimise (waves of CTAs) x (rounds per CTA + one round of fixed cost: tables, TMEM, epilogue).
cudaError_t launch_gemm_tc48(const llvq_codec *c, Dec48::Args a, const llvq_weight *w, const void *X, int batch,
                             float *Y, cudaStream_t st) {
    const int mt = (w->rows + kTcRows - 1) / kTcRows;
    const int nrounds = (w->blocks_per_row + kTc48Slots - 1) / kTc48Slots;
    int best_rps = nrounds;
    long long best_cost = -1;
    for (int sp = 1; sp <= nrounds; sp++) {
        const int rps = (nrounds + sp - 1) / sp;
        const int splits = (nrounds + rps - 1) / rps;
        const long long waves = ((long long)mt * splits + c->num_sms - 1) / c->num_sms;
        const long long cost = waves * (rps + 1);
        if (best_cost < 0 || cost < best_cost) { best_cost = cost; best_rps = rps; }
    }
    const int splits = std::max(1, (nrounds + best_rps - 1) / best_rps);
    cudaError_t e = cudaMemsetAsync(Y, 0, (size_t)batch * w->rows * sizeof(float), st);
    if (e != cudaSuccess) return e;
    k_gemm_tc48<<<dim3(mt, splits), kTc48Threads, tc48_smem_bytes(), st>>>(
        a, (const SmemEven48 *)c->d_even48, c->d_tabC48, (const unsigned long long *)w->words, w->row_pitch_words,
        w->rows, w->blocks_per_row, batch, w->gain_mode, (const __half *)w->gains, (const __half *)X, Y, best_rps,
        c->d_flags, g_first_wait_tries.load(), g_mma_wait_tries.load());
    return cudaGetLastError();
}

template <class D>
cudaError_t gemm_dispatch(const llvq_codec *c, typename D::Args a, const llvq_weight *w, const void *X,
                          int batch, float *Y, cudaStream_t s) {
    if (batch >= kTensorCoreMinBatch) {
        // 48 bits: tensor cores.  72/96 bits: the decode dominates, and the CUDA-core product that
        // decodes each block once for the whole batch is faster than 128-row tensor-core rounds
        if constexpr (std::is_same<D, Dec48>::value) return launch_gemm_tc48(c, a, w, X, batch, Y, s);
        else if (batch == 8) return launch_gemm<D, 8>(c, a, w, X, Y, s);
        else return launch_gemm<D, 16>(c, a, w, X, Y, s, batch);
    }
    if constexpr (std::is_same<D, Dec48>::value) {
        // long row ranges (>= kWarpBinnedMinBlocks blocks per SM) at batch 1 and 2: the warp-binned
        // kernel; shorter ranges and larger batches: the coset-sorted kernel (measured on B200)
        const long long per_sm = (long long)((w->rows + c->num_sms - 1) / c->num_sms) * w->blocks_per_row;
        if (per_sm >= kWarpBinnedMinBlocks && batch <= 2)
            return batch == 1 ? launch_gemv48<1>(c, a, w, X, Y, s) : launch_gemv48<2>(c, a, w, X, Y, s);
        switch (batch) {
            case 1: return launch_gemm_bin48<1>(c, a, w, X, Y, s);
            case 2: return launch_gemm_bin48<2>(c, a, w, X, Y, s);
            case 3: return launch_gemm_bin48<3>(c, a, w, X, Y, s);
            case 4: return launch_gemm_bin48<4>(c, a, w, X, Y, s);
            case 5: return launch_gemm_bin48<5>(c, a, w, X, Y, s);
            case 6: return launch_gemm_bin48<6>(c, a, w, X, Y, s);
            default: return launch_gemm_bin48<7>(c, a, w, X, Y, s);
        }
    } else {
        switch (batch) {
            case 1: return launch_gemm<D, 1>(c, a, w, X, Y, s);
            case 2: return launch_gemm<D, 2>(c, a, w, X, Y, s);
            case 3: return launch_gemm<D, 3>(c, a, w, X, Y, s);
            case 4: return launch_gemm<D, 4>(c, a, w, X, Y, s);
            case 5: return launch_gemm<D, 5>(c, a, w, X, Y, s);
            case 6: return launch_gemm<D, 6>(c, a, w, X, Y, s);
            default: return launch_gemm<D, 7>(c, a, w, X, Y, s);
        }
    }
}

llvq_status check_weight(const llvq_codec *c, const llvq_weight *w) {
    if (!w || !w->words || !w->gains) return LLVQ_ERR_ARG;
    if (w->rows < 0 || w->cols < 0 || w->blocks_per_row < 0) return LLVQ_ERR_ARG;
    if (w->blocks_per_row != (w->cols + 23) / 24) return LLVQ_ERR_ARG;
    if (w->row_pitch_words < w->blocks_per_row) return LLVQ_ERR_ARG;
    if (w->index_bits != c->index_bits) return LLVQ_ERR_ARG;
    if (w->word_bytes != (c->index_bits == 48 ? 8 : 16)) return LLVQ_ERR_ARG;
    if (w->gain_mode != LLVQ_GAIN_FP16_DIRECT && w->gain_mode != LLVQ_GAIN_U8_TABLE) return LLVQ_ERR_ARG;
    if (!aligned(w->words, (size_t)w->word_bytes) || !aligned(w->gains, 2)) return LLVQ_ERR_ARG;
    return LLVQ_OK;
}

}  // namespace

// ---- decode without any device allocation -----------------------------------------------
// A caller that cannot allocate device memory (under a framework's memory pool that owns every
// byte, in a plug-in with a fixed device budget, on a path where cudaMalloc's device-wide
// synchronisation is not allowed) cannot create a codec, because llvq_codec_create allocates its
// tables with cudaMalloc.  llvq_decode_noalloc keeps the decode kernel's non-input, non-output
// global memory -- the 48-bit table image and the status word -- in this file-scope device array
// instead.  Every GPU that loads the library holds it (kNoAllocScratchBytes) until the process
// exits.
constexpr size_t kNoAllocFlagOffset = (sizeof(Smem48) + 255) / 256 * 256;
constexpr size_t kNoAllocScratchBytes = kNoAllocFlagOffset + 256;     // 76,544 B
static_assert(kNoAllocScratchBytes == 76544, "the documented size of the allocation-free decode's array");
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
unsigned char *g_noalloc_ptr[kNoAllocMaxDevices] = {};   // device address of the array, per device
unsigned long long g_noalloc_npoints = 0;

// Once per device, with that device current: build the 48-bit table image on the host, find the
// array's device address and copy the image in (synchronous; no allocation on the device).
llvq_status noalloc_setup(int dev, unsigned char **out) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev]) { *out = g_noalloc_ptr[dev]; return LLVQ_OK; }
    HostTables T;
    std::string err;
    if (!build_host_tables(48, T, err)) { g_last_error = err; return LLVQ_ERR_UNSUPPORTED; }
    std::vector<unsigned char> image(sizeof(Smem48));
    const llvq_status st = build_image48(T, *reinterpret_cast<Smem48 *>(image.data()), err);
    if (st != LLVQ_OK) { g_last_error = err; return st; }
    unsigned char *ptr = nullptr;
    if (cudaGetSymbolAddress((void **)&ptr, g_noalloc_scratch) != cudaSuccess || !ptr ||
        cudaMemcpy(ptr, image.data(), image.size(), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaFuncSetAttribute(k_decode<Dec48>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem48)) !=
            cudaSuccess) {
        cudaGetLastError();
        return LLVQ_ERR_CUDA;
    }
    g_noalloc_npoints = (unsigned long long)T.n_points;
    g_noalloc_ptr[dev] = ptr;
    *out = ptr;
    return LLVQ_OK;
}
void set_kernel_attrs() {
    static std::once_flag once;
    std::call_once(once, [] {
        cudaFuncSetAttribute(k_decode<Dec48>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem48));
        cudaFuncSetAttribute(k_decode<Dec72>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem72));
        set_bin48_attrs(std::make_integer_sequence<int, 7>{});
        set_gemv48_attrs(std::make_integer_sequence<int, 2>{});
        cudaFuncSetAttribute(k_encode48, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(EncSmem48));
        cudaFuncSetAttribute(k_search48<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(SearchSmem48));
        cudaFuncSetAttribute(k_search48<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(SearchSmem48));
        cudaFuncSetAttribute(k_encode72, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(EncSmem72));
        cudaFuncSetAttribute(k_encode96, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(EncSmem96));
        cudaFuncSetAttribute(k_gemm_tc48, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc48_smem_bytes());
        set_gemm_attrs<Dec72>(std::make_integer_sequence<int, kTensorCoreMinBatch - 1>{});
        cudaFuncSetAttribute(k_decode<Dec96>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem96));
        set_gemm_attrs<Dec96>(std::make_integer_sequence<int, kTensorCoreMinBatch - 1>{});
    });
}

llvq_status codec_create96(llvq_codec **out) {
    llvq_codec *c = new llvq_codec;
    c->index_bits = 96;
    std::vector<unsigned char> image;
    std::string err;
    llvq_status st = LLVQ_OK;
    if (cudaGetDevice(&c->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess) {
        err = "no CUDA device";
        st = LLVQ_ERR_CUDA;
    }
    if (st == LLVQ_OK) st = create96(c, image, err);
    if (st == LLVQ_OK &&
        !(cudaMalloc(&c->d_image, image.size()) == cudaSuccess &&
          cudaMemcpy(c->d_image, image.data(), image.size(), cudaMemcpyHostToDevice) == cudaSuccess &&
          cudaMalloc(&c->d_flags, sizeof(unsigned)) == cudaSuccess &&
          cudaMemset(c->d_flags, 0, sizeof(unsigned)) == cudaSuccess)) {
        err = "device allocation for the 96-bit codec failed";
        st = LLVQ_ERR_CUDA;
    }
    if (st != LLVQ_OK) {
        cudaGetLastError();
        g_last_error = err;
        llvq_codec_destroy(c);
        return st;
    }
    set_kernel_attrs();
    *out = c;
    return LLVQ_OK;
}

}  // namespace

extern "C" {

llvq_status llvq_decode_noalloc(int32_t index_bits, const void *d_words, int32_t word_bytes, int64_t n,
                                int8_t *d_out, void *stream) {
    if (index_bits != 48) {
        g_last_error = "llvq_decode_noalloc holds only the 48-bit table image (76,544 bytes); larger budgets need a codec";
        return LLVQ_ERR_UNSUPPORTED;
    }
    if (n < 0 || word_bytes != 8) return LLVQ_ERR_ARG;
    if (n == 0) return LLVQ_OK;
    if (!d_words || !d_out || !aligned(d_words, 8) || !aligned(d_out, 8)) return LLVQ_ERR_ARG;
    int dev = -1, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return LLVQ_ERR_CUDA;
    unsigned char *ptr = nullptr;
    const llvq_status st = noalloc_setup(dev, &ptr);
    if (st != LLVQ_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned *flags = reinterpret_cast<unsigned *>(ptr + kNoAllocFlagOffset);
    if (cudaMemsetAsync(flags, 0, sizeof(unsigned), s) != cudaSuccess) return LLVQ_ERR_CUDA;
    const int threads = 512;
    const long long want = (n + threads - 1) / threads;
    const int grid = (int)std::max(1LL, std::min(want, (long long)nsm * Dec48::kCtasPerSm));
    k_decode<Dec48><<<grid, threads, sizeof(Smem48), s>>>(
        Dec48::Args{reinterpret_cast<const Smem48 *>(ptr), g_noalloc_npoints},
        (const Dec48::Word *)d_words, n, d_out, flags);
    return cudaGetLastError() == cudaSuccess ? LLVQ_OK : LLVQ_ERR_CUDA;
}


const char *llvq_last_error_message(void) { return g_last_error.c_str(); }

void llvq_set_wait_polls(uint32_t table_polls, uint32_t mma_polls) {
    g_first_wait_tries.store(table_polls == 0xFFFFFFFFu ? kBulkWaitTries : table_polls);
    g_mma_wait_tries.store(mma_polls == 0xFFFFFFFFu ? kMmaWaitTries : mma_polls);
}

llvq_status llvq_class_table96(int32_t m, llvq_class96 *out, int64_t capacity, int64_t *n_classes) {
    static_assert(sizeof(llvq_class96) == sizeof(Rec96), "llvq_class96 mirrors Rec96");
    static std::mutex mu;
    static std::unique_ptr<Tables96> tables;
    std::lock_guard<std::mutex> g(mu);
    if (!tables) {
        auto t = std::make_unique<Tables96>();
        std::string err;
        if (!build_tables96(*t, std::max(1, (int)std::thread::hardware_concurrency()), err)) {
            g_last_error = err;
            return LLVQ_ERR_UNSUPPORTED;
        }
        tables = std::move(t);
    }
    if (m < 2 || m > tables->M) return LLVQ_ERR_ARG;
    const int64_t n = tables->shell_classes[m];
    if (n_classes) *n_classes = n;
    if (!out) return LLVQ_OK;
    if (capacity < n) return LLVQ_ERR_ARG;
    std::vector<Rec96> buf((size_t)n);
    std::string err;
    if (!fill_shell96(*tables, m, buf.data(), err)) {
        g_last_error = err;
        return LLVQ_ERR_UNSUPPORTED;
    }
    std::memcpy(out, buf.data(), buf.size() * sizeof(Rec96));
    return LLVQ_OK;
}

const char *llvq_status_string(llvq_status s) {
    switch (s) {
        case LLVQ_OK: return "ok";
        case LLVQ_ERR_ARG: return "invalid argument";
        case LLVQ_ERR_UNSUPPORTED: return "unsupported";
        case LLVQ_ERR_CUDA: return "CUDA error";
        case LLVQ_ERR_DEVICE_FLAG: return "device flag raised";
    }
    return "unknown status";
}

llvq_status llvq_codec_create(int32_t index_bits, llvq_codec **out) {
    if (!out) return LLVQ_ERR_ARG;
    *out = nullptr;
    if (index_bits != 48 && index_bits != 72 && index_bits != 96) return LLVQ_ERR_UNSUPPORTED;
    if (index_bits == 96) return codec_create96(out);
    HostTables T;
    std::string err;
    if (!build_host_tables(index_bits, T, err)) { g_last_error = err; return LLVQ_ERR_UNSUPPORTED; }
    std::vector<unsigned char> image;
    std::vector<Rec72> recs;
    std::vector<uint32_t> guide, tabC;
    std::vector<unsigned char> even(sizeof(SmemEven48));
    std::vector<unsigned char> gv(sizeof(SmemGv48));
    std::vector<unsigned char> enc(sizeof(EncSmem48));
    std::unique_ptr<SearchImage48> search_image(new SearchImage48);
    std::vector<unsigned char> enc72(sizeof(EncSmem72));
    std::vector<unsigned long long> keys72;
    llvq_status st;
    if (index_bits == 48) {
        image.resize(sizeof(Smem48));
        st = build_image48(T, *reinterpret_cast<Smem48 *>(image.data()), err);
        if (st == LLVQ_OK)
            st = build_even48(T, *reinterpret_cast<Smem48 *>(image.data()), *reinterpret_cast<SmemEven48 *>(even.data()),
                              tabC, err);
        if (st == LLVQ_OK)
            st = build_gv48(T, *reinterpret_cast<const Smem48 *>(image.data()), *reinterpret_cast<const SmemEven48 *>(even.data()),
                            *reinterpret_cast<SmemGv48 *>(gv.data()), err);
        if (st == LLVQ_OK) st = build_enc48(T, *reinterpret_cast<EncSmem48 *>(enc.data()), err);
        if (st == LLVQ_OK) st = build_search48(T, *search_image, err);
    } else {
        image.resize(sizeof(Smem72));
        st = build_image72(T, *reinterpret_cast<Smem72 *>(image.data()), recs, guide, err);
        if (st == LLVQ_OK) st = build_enc72(T, *reinterpret_cast<EncSmem72 *>(enc72.data()), keys72, err);
    }
    if (st != LLVQ_OK) { g_last_error = err; return st; }
    llvq_codec *c = new llvq_codec;
    c->index_bits = index_bits;
    c->M = T.M;
    c->npoints = T.n_points;
    c->nclasses = (int64_t)T.classes.size();
    bool okc = cudaGetDevice(&c->device) == cudaSuccess &&
               cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) == cudaSuccess &&
               cudaMalloc(&c->d_image, image.size()) == cudaSuccess &&
               cudaMemcpy(c->d_image, image.data(), image.size(), cudaMemcpyHostToDevice) == cudaSuccess &&
               cudaMalloc(&c->d_flags, sizeof(unsigned)) == cudaSuccess &&
               cudaMemset(c->d_flags, 0, sizeof(unsigned)) == cudaSuccess;
    if (okc && index_bits == 48) {
        okc = cudaMalloc(&c->d_enc48, enc.size()) == cudaSuccess &&
              cudaMemcpy(c->d_enc48, enc.data(), enc.size(), cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMalloc(&c->d_even48, even.size()) == cudaSuccess &&
              cudaMemcpy(c->d_even48, even.data(), even.size(), cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMalloc(&c->d_tabC48, std::max<size_t>(tabC.size(), 1) * sizeof(uint32_t)) == cudaSuccess &&
              cudaMemcpy(c->d_tabC48, tabC.data(), tabC.size() * sizeof(uint32_t), cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMalloc(&c->d_gv48, gv.size()) == cudaSuccess &&
              cudaMemcpy(c->d_gv48, gv.data(), gv.size(), cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMalloc(&c->d_search48, sizeof(SearchImage48)) == cudaSuccess &&
              cudaMemcpy(c->d_search48, search_image.get(), sizeof(SearchImage48), cudaMemcpyHostToDevice) == cudaSuccess;
    }
    if (okc && index_bits == 72) {
        okc = cudaMalloc(&c->d_recs72, recs.size() * sizeof(Rec72)) == cudaSuccess &&
              cudaMemcpy(c->d_recs72, recs.data(), recs.size() * sizeof(Rec72), cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMalloc(&c->d_enc72, enc72.size()) == cudaSuccess &&
              cudaMemcpy(c->d_enc72, enc72.data(), enc72.size(), cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMalloc(&c->d_keys72, keys72.size() * sizeof(unsigned long long)) == cudaSuccess &&
              cudaMemcpy(c->d_keys72, keys72.data(), keys72.size() * sizeof(unsigned long long),
                         cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMalloc(&c->d_guide72, guide.size() * sizeof(uint32_t)) == cudaSuccess &&
              cudaMemcpy(c->d_guide72, guide.data(), guide.size() * sizeof(uint32_t), cudaMemcpyHostToDevice) == cudaSuccess;
    }
    if (!okc) {
        cudaGetLastError();
        llvq_codec_destroy(c);
        return LLVQ_ERR_CUDA;
    }
    set_kernel_attrs();
    *out = c;
    return LLVQ_OK;
}

void llvq_codec_destroy(llvq_codec *c) {
    if (!c) return;
    if (c->d_image) cudaFree(c->d_image);
    if (c->d_recs72) cudaFree(c->d_recs72);
    if (c->d_guide72) cudaFree(c->d_guide72);
    if (c->d_recs96) cudaFree(c->d_recs96);
    if (c->d_guide96) cudaFree(c->d_guide96);
    if (c->d_flags) cudaFree(c->d_flags);
    if (c->d_even48) cudaFree(c->d_even48);
    if (c->d_enc48) cudaFree(c->d_enc48);
    if (c->d_enc72) cudaFree(c->d_enc72);
    if (c->d_keys72) cudaFree(c->d_keys72);
    if (c->d_enc96) cudaFree(c->d_enc96);
    if (c->d_keys96) cudaFree(c->d_keys96);
    if (c->d_tabC48) cudaFree(c->d_tabC48);
    if (c->d_gv48) cudaFree(c->d_gv48);
    if (c->d_search48) cudaFree(c->d_search48);

    delete c;
}

llvq_status llvq_codec_info(const llvq_codec *c, int32_t *max_shell, uint64_t *lo, uint64_t *hi,
                            int64_t *n_classes) {
    if (!c) return LLVQ_ERR_ARG;
    if (max_shell) *max_shell = c->M;
    if (lo) *lo = (uint64_t)c->npoints;
    if (hi) *hi = (uint64_t)(c->npoints >> 64);
    if (n_classes) *n_classes = c->nclasses;
    return LLVQ_OK;
}

llvq_status llvq_decode(const llvq_codec *c, const void *d_words, int32_t word_bytes, int64_t n,
                        int8_t *d_out, void *stream) {
    if (!c || n < 0) return LLVQ_ERR_ARG;
    if (n == 0) return LLVQ_OK;
    if (!d_words || !d_out) return LLVQ_ERR_ARG;
    if (word_bytes != (c->index_bits == 48 ? 8 : 16)) return LLVQ_ERR_ARG;
    if (!aligned(d_words, (size_t)word_bytes) || !aligned(d_out, 8)) return LLVQ_ERR_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const cudaError_t e = c->index_bits == 48   ? launch_decode<Dec48>(c, args48(c), d_words, n, d_out, st)
                          : c->index_bits == 72 ? launch_decode<Dec72>(c, args72(c), d_words, n, d_out, st)
                                                : launch_decode<Dec96>(c, args96(c), d_words, n, d_out, st);
    return e == cudaSuccess ? LLVQ_OK : LLVQ_ERR_CUDA;
}

llvq_status llvq_encode(const llvq_codec *c, const int8_t *d_vectors, int64_t n, void *d_words, int32_t word_bytes,
                        void *stream) {
    if (!c || n < 0) return LLVQ_ERR_ARG;
    if (n == 0) return LLVQ_OK;
    if (!d_vectors || !d_words || word_bytes != (c->index_bits == 48 ? 8 : 16)) return LLVQ_ERR_ARG;
    if (!aligned(d_vectors, 8) || !aligned(d_words, (size_t)word_bytes)) return LLVQ_ERR_ARG;
    const int threads = 512;
    const long long want = (n + threads - 1) / threads;
    const int grid = (int)std::max(1LL, std::min(want, (long long)c->num_sms * 2));
    if (c->index_bits == 48)
        k_encode48<<<grid, threads, sizeof(EncSmem48), (cudaStream_t)stream>>>(
            (const EncSmem48 *)c->d_enc48, (unsigned long long)c->npoints, d_vectors, n,
            (unsigned long long *)d_words, c->d_flags);
    else if (c->index_bits == 72)
        k_encode72<<<grid, threads, sizeof(EncSmem72), (cudaStream_t)stream>>>(
            (const EncSmem72 *)c->d_enc72, c->d_recs72, c->d_keys72, (unsigned long long)c->npoints,
            (unsigned long long)(c->npoints >> 64), d_vectors, n, (ulonglong2 *)d_words, c->d_flags);
    else {
        const long long want96 = (n + 255) / 256;
        const int grid96 = (int)std::max(1LL, std::min(want96, (long long)c->num_sms * 4));
        k_encode96<<<grid96, 256, sizeof(EncSmem96), (cudaStream_t)stream>>>(
            (const EncSmem96 *)c->d_enc96, c->d_recs96, c->d_keys96, (unsigned long long)c->npoints,
            (unsigned long long)(c->npoints >> 64), d_vectors, n, (ulonglong2 *)d_words, c->d_flags);
    }
    return cudaGetLastError() == cudaSuccess ? LLVQ_OK : LLVQ_ERR_CUDA;
}

llvq_status llvq_gemm_smallbatch(const llvq_codec *c, const llvq_weight *w, const void *d_X,
                                 int32_t batch, float *d_Y, void *stream) {
    if (!c) return LLVQ_ERR_ARG;
    const llvq_status st = check_weight(c, w);
    if (st != LLVQ_OK) return st;
    if (batch < 1 || batch > 16 || !d_X || !d_Y) return LLVQ_ERR_ARG;
    if (!aligned(d_X, 16) || !aligned(d_Y, 4)) return LLVQ_ERR_ARG;
    if (w->rows == 0) return LLVQ_OK;
    cudaStream_t s = (cudaStream_t)stream;
    const cudaError_t e = c->index_bits == 48   ? gemm_dispatch<Dec48>(c, args48(c), w, d_X, batch, d_Y, s)
                          : c->index_bits == 72 ? gemm_dispatch<Dec72>(c, args72(c), w, d_X, batch, d_Y, s)
                                                : gemm_dispatch<Dec96>(c, args96(c), w, d_X, batch, d_Y, s);
    return e == cudaSuccess ? LLVQ_OK : LLVQ_ERR_CUDA;
}

llvq_status llvq_gemv(const llvq_codec *c, const llvq_weight *w, const void *d_x, float *d_y,
                      void *stream) {
    return llvq_gemm_smallbatch(c, w, d_x, 1, d_y, stream);
}

llvq_status llvq_search(const llvq_codec *c, int32_t max_shell, int32_t mode, double scale, const float *d_X,
                        int64_t n, int8_t *d_points, double *d_dots, const double *d_gain_levels,
                        int32_t n_levels, uint8_t *d_gain_codes, void *stream) {
    if (!c || n < 0) return LLVQ_ERR_ARG;
    if (c->index_bits != 48) return LLVQ_ERR_UNSUPPORTED;
    if (max_shell < 2 || max_shell > c->M) return LLVQ_ERR_ARG;
    if (mode != LLVQ_SEARCH_ANGULAR && mode != LLVQ_SEARCH_EUCLIDEAN) return LLVQ_ERR_ARG;
    if (mode == LLVQ_SEARCH_EUCLIDEAN && !(std::isfinite(scale) && scale > 0.0)) return LLVQ_ERR_ARG;
    const bool gains = n_levels != 0 || d_gain_levels || d_gain_codes;
    if (gains && (mode != LLVQ_SEARCH_ANGULAR || n_levels < 1 || n_levels > 256 || !d_gain_levels || !d_gain_codes ||
                  !aligned(d_gain_levels, 8)))
        return LLVQ_ERR_ARG;
    if (n == 0) return LLVQ_OK;
    if (!d_X || !d_points || !aligned(d_X, 4) || (d_dots && !aligned(d_dots, 8))) return LLVQ_ERR_ARG;
    SearchArgs48 a;
    a.image = (const SearchImage48 *)c->d_search48;
    a.max_shell = max_shell;
    a.mode = mode;
    a.scale = scale;
    a.X = d_X;
    a.n = n;
    a.points = d_points;
    a.dots = d_dots;
    a.levels = gains ? d_gain_levels : nullptr;
    a.n_levels = gains ? n_levels : 0;
    a.codes = gains ? d_gain_codes : nullptr;
    a.flags = c->d_flags;
    search_list_prefixes(max_shell, a.nal);
    // one CTA per vector, one resident per SM
    const long long grid = std::min<long long>(n, (long long)c->num_sms);
    if (mode == LLVQ_SEARCH_ANGULAR)
        k_search48<0><<<(int)grid, kSrThreads, sizeof(SearchSmem48), (cudaStream_t)stream>>>(a);
    else
        k_search48<1><<<(int)grid, kSrThreads, sizeof(SearchSmem48), (cudaStream_t)stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? LLVQ_OK : LLVQ_ERR_CUDA;
}

static size_t gptq_align(size_t x) { return (x + 255) & ~(size_t)255; }

size_t llvq_spherical_gptq_workspace(int32_t rows, int32_t cols) {
    if (rows < 0 || rows > 65535 || cols <= 0 || cols % 24) return 0;
    const size_t nb = (size_t)cols / 24, r = (size_t)rows;
    return gptq_align(nb * 24 * (size_t)cols * sizeof(double)) + gptq_align(r * 24 * sizeof(float)) +
           gptq_align(r * 24) + gptq_align(r * 24 * sizeof(double));
}

llvq_status llvq_spherical_gptq(const llvq_codec *c, int32_t max_shell, int32_t rows, int32_t cols, double *d_W,
                                const double *d_U, int8_t *d_points, double *d_norms, void *d_workspace,
                                size_t workspace_bytes, void *stream) {
    if (!c) return LLVQ_ERR_ARG;
    if (c->index_bits != 48) return LLVQ_ERR_UNSUPPORTED;
    if (max_shell < 2 || max_shell > c->M || rows < 0 || rows > 65535 || cols <= 0 || cols % 24) return LLVQ_ERR_ARG;
    if (rows == 0) return LLVQ_OK;
    if (!d_W || !d_U || !d_points || !d_norms || !d_workspace || !aligned(d_W, 8) || !aligned(d_U, 8) ||
        !aligned(d_norms, 8) || !aligned(d_workspace, 256) || workspace_bytes < llvq_spherical_gptq_workspace(rows, cols))
        return LLVQ_ERR_ARG;
    const int nb = cols / 24;
    unsigned char *ws = (unsigned char *)d_workspace;
    double *G = (double *)ws;
    ws += gptq_align((size_t)nb * 24 * cols * sizeof(double));
    float *Xf = (float *)ws;
    ws += gptq_align((size_t)rows * 24 * sizeof(float));
    int8_t *P = (int8_t *)ws;
    ws += gptq_align((size_t)rows * 24);
    double *E = (double *)ws;
    cudaStream_t s = (cudaStream_t)stream;
    k_gptq_gmat<<<dim3((cols + kGqThreads - 1) / kGqThreads, nb), kGqThreads, 0, s>>>(d_U, G, cols);
    SearchArgs48 a;
    a.image = (const SearchImage48 *)c->d_search48;
    a.max_shell = max_shell;
    a.mode = LLVQ_SEARCH_ANGULAR;
    a.scale = 1.0;
    a.X = Xf;
    a.n = rows;
    a.points = P;
    a.dots = nullptr;
    a.levels = nullptr;
    a.n_levels = 0;
    a.codes = nullptr;
    a.flags = c->d_flags;
    search_list_prefixes(max_shell, a.nal);
    const int sgrid = std::min(rows, c->num_sms);
    for (int b = 0; b < nb; b++) {
        k_gptq_gather<<<(rows * 24 + 255) / 256, 256, 0, s>>>(d_W, Xf, rows, cols, b);
        k_search48<0><<<sgrid, kSrThreads, sizeof(SearchSmem48), s>>>(a);
        k_gptq_retract<<<(rows + 127) / 128, 128, 0, s>>>(d_W, P, E, d_points, d_norms, rows, cols, b);
        const int rest = cols - 24 * (b + 1);
        if (rest > 0) k_gptq_update<<<dim3((rest + kGqThreads - 1) / kGqThreads, rows), kGqThreads, 0, s>>>(d_W, E, G, cols, b);
    }
    return cudaGetLastError() == cudaSuccess ? LLVQ_OK : LLVQ_ERR_CUDA;
}

llvq_status llvq_get_error(const llvq_codec *c, void *stream, uint32_t *flags) {
    if (!c || !flags) return LLVQ_ERR_ARG;
    unsigned h = 0;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess ||
        cudaMemcpy(&h, c->d_flags, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(c->d_flags, 0, sizeof(unsigned)) != cudaSuccess) {
        return LLVQ_ERR_CUDA;
    }
    *flags = h;
    return h ? LLVQ_ERR_DEVICE_FLAG : LLVQ_OK;
}

}  // extern "C"
