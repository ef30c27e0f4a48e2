// encode48.cuh -- the inverse map for the 48-bit budget: a Leech lattice point (int8 [24],
// sqrt(8)-scaled coordinates) to its packed index, one thread per vector.
//
// "Leech Lattice Vector Quantization for Efficient LLM Compression", papernotes.org notes,
// 方法详解 / 关键设计 2: the index is the shell offset plus the class offset plus
// r + A (s + 2^B I''), and the pages describe the conversion in both directions.  Steps:
//   1. membership: all coordinates of one parity; even: {i: x_i = 2 mod 4} is a codeword and
//      sum x = 0 (mod 8); odd: {i: x_i = 1 mod 4} is a codeword and sum x = 4 (mod 8);
//      shell m = sum x^2 / 16 in 2..13;
//   2. class: the multiset of |x_i| as a count vector packed 5 bits per magnitude, the largest
//      magnitude most significant, so that the classes of one shell and coset (ordered by their
//      descending magnitude tuples) are in ascending key order: a binary search;
//   3. r: the codeword's place among all codewords in ascending mask order (odd) or among those
//      of its weight (even).  Coordinates 12..23 form an information set of this code (checked
//      when the tables are built), so the codewords' top 12 bits are distinct and ascend with the
//      mask: the place in mask order is the top 12 bits, one lookup confirms the codeword, and a
//      4096-entry table gives the place within the weight;
//   4. s (even): bit j = sign of the j-th nonzero coordinate (ascending) with the highest
//      coordinate of S skipped (its sign is the parity sign);
//   5. I'': the lexicographic ranks p_S of the magnitudes on S (ascending positions) and p_C of
//      those off S, I'' = p_S + P_S p_C (odd: one rank over all 24 positions), with exact 64-bit
//      integer arithmetic: rank += M c_<g / L, M <- M c_g / L (M = arrangements left).
// A vector that is not a coded point gets the index 2^48 - 1 (>= N_M; it decodes to zero) and
// raises LLVQ_FLAG_NOT_CODED.
#pragma once
#include "device_common.cuh"

namespace llvq {

constexpr int kEncClasses48 = 384;
constexpr int kEncShells48 = 16;
constexpr unsigned long long kEncInvalid48 = (1ull << 48) - 1ull;

struct alignas(16) EncSmem48 {
    uint32_t golay_mask[4096];                    // ascending mask
    uint32_t golay_weight[4096];                  // ascending (weight, mask)
    unsigned long long key_lo[kEncClasses48];     // counts of |x| = 0..11, 5 bits each
    uint32_t key_hi[kEncClasses48];               // counts of |x| = 12, 13
    uint32_t info[kEncClasses48];                 // A | B << 13 | odd << 18 | k << 19
    unsigned long long start[kEncClasses48];      // first global index of the class
    unsigned long long P0[kEncClasses48];         // arrangements of set 0 (odd: all; even: off S)
    unsigned long long P1[kEncClasses48];         // arrangements of set 1 (even: on S; odd: 1)
    unsigned long long vals0[kEncClasses48];      // bytes: magnitudes of the set-0 groups, ascending (0xFF unused)
    uint32_t vals1[kEncClasses48];                // bytes: magnitudes of the set-1 groups, ascending (0xFF unused)
    unsigned long long cnt0[kEncClasses48];       // bytes: counts of the set-0 groups
    uint32_t cnt1[kEncClasses48];                 // bytes: counts of the set-1 groups
    unsigned long long mL[32];                    // ceil(2^64 / L), L = 2..24
    uint16_t seg_first[kEncShells48][2];          // classes of (shell, coset): first index
    uint16_t seg_count[kEncShells48][2];          //                            and count
    uint16_t wbase[32];                           // first by-weight slot of weight k
    uint16_t wrank[4096];                         // codeword with top 12 bits t: place within its weight
};
static_assert(sizeof(EncSmem48) % 16 == 0, "16-byte table image");

// number of bytes of v (8 bytes) that are below a
__device__ __forceinline__ uint32_t count_below8(unsigned long long v, uint32_t a) {
    const uint32_t aa = a * 0x01010101u;
    return (uint32_t)__popc(__vcmpltu4((uint32_t)v, aa) & 0x01010101u) +
           (uint32_t)__popc(__vcmpltu4((uint32_t)(v >> 32), aa) & 0x01010101u);
}

// sum of the bytes of c (8 bytes) below byte index g, and byte g itself
__device__ __forceinline__ void cum_and_count8(unsigned long long c, uint32_t g, uint32_t &below, uint32_t &at) {
    const unsigned long long keep = g >= 8u ? ~0ull : ((1ull << (8u * g)) - 1ull);
    const unsigned long long lo = c & keep;
    below = (uint32_t)__dp4a((uint32_t)lo, 0x01010101u, __dp4a((uint32_t)(lo >> 32), 0x01010101u, 0u));
    at = (uint32_t)(c >> (8u * (g & 7u))) & 0xFFu;
}

// exact M * n / L for a product divisible by L (M n < 2^40): multiply-high by ceil(2^64 / L)
__device__ __forceinline__ unsigned long long exact_div_small(unsigned long long Mn, uint32_t L,
                                                              const unsigned long long *mL) {
    return L == 1u ? Mn : __umul64hi(Mn, mL[L]);
}

__device__ __forceinline__ bool encode48(const uint32_t xw[6], const EncSmem48 &E, unsigned long long npoints,
                                         unsigned long long &index) {
    index = kEncInvalid48;
    // 1. magnitudes, parity, norm, sum
    uint32_t a[6];
    int norm = 0, sum = 0;
    const bool odd = xw[0] & 1u;
    bool ok = true;
#pragma unroll
    for (int q = 0; q < 6; q++) {
        a[q] = __vabsss4(xw[q]);
        ok &= (xw[q] & 0x01010101u) == (odd ? 0x01010101u : 0u);
        norm = __dp4a((int)a[q], (int)a[q], norm);
        sum = __dp4a((int)xw[q], 0x01010101, sum);
    }
    const int m = norm >> 4;
    ok &= (norm & 15) == 0 && m >= 2 && m < kEncShells48 && ((sum & 7) == (odd ? 4 : 0));
    // codeword mask: even -> |x| = 2 mod 4; odd -> x = 1 mod 4
    uint32_t word = 0, nz = 0, neg = 0;
#pragma unroll
    for (int q = 0; q < 6; q++) {
        const uint32_t w = odd ? __vcmpeq4(xw[q] & 0x03030303u, 0x01010101u)
                               : __vcmpeq4(a[q] & 0x03030303u, 0x02020202u);
        word |= bytes_to_nibble(w) << (4 * q);
        nz |= bytes_to_nibble(__vcmpne4(a[q], 0u)) << (4 * q);
        neg |= bytes_to_nibble((xw[q] >> 7) & 0x01010101u) << (4 * q);
    }
    // 2. class key: 5-bit count per magnitude (|x| <= 13 in the coded shells)
    unsigned long long klo = 0;
    uint32_t khi = 0;
#pragma unroll
    for (int i = 0; i < 24; i++) {
        const uint32_t v = (a[i >> 2] >> (8 * (i & 3))) & 0xFFu;
        ok &= v <= 13u;
        if (v < 12u) klo += 1ull << (5u * v);
        else khi += 1u << (5u * ((v - 12u) & 1u));
    }
    if (!ok) return false;
    const int first = E.seg_first[m][odd], cnt = E.seg_count[m][odd];
    int l = first, h = first + cnt - 1;
    while (l < h) {                                      // first class with key >= the vector's
        const int mid = (l + h) >> 1;
        const bool less = E.key_hi[mid] < khi || (E.key_hi[mid] == khi && E.key_lo[mid] < klo);
        if (less) l = mid + 1; else h = mid;
    }
    if (cnt == 0 || E.key_hi[l] != khi || E.key_lo[l] != klo) return false;
    const int cls = l;
    const uint32_t info = E.info[cls];
    const uint32_t A = info & 0x1FFFu, B = (info >> 13) & 0x1Fu, k = (info >> 19) & 0x1Fu;
    // 3. r
    const uint32_t t12 = word >> 12;
    if (E.golay_mask[t12] != word || (!odd && (uint32_t)__popc(word) != k)) return false;
    const uint32_t r = odd ? t12 : E.wrank[t12];
    // 4. s (even): signs of the nonzero coordinates, ascending, skipping the top of S
    uint32_t s = 0;
    if (!odd) {
        const uint32_t top = word ? (0x80000000u >> __clz(word)) : 0u;
        uint32_t msk = nz & ~top, j = 0;
        while (msk) {
            const uint32_t b = msk & (0u - msk);
            s |= (neg & b) ? (1u << j) : 0u;
            j++;
            msk ^= b;
        }
    }
    // 5. arrangement ranks: set 0 = off S (odd: all positions), set 1 = on S
    const uint32_t mask1 = odd ? 0u : word;
    unsigned long long M0 = E.P0[cls], M1 = E.P1[cls], rk0 = 0, rk1 = 0;
    unsigned long long c0 = E.cnt0[cls];
    uint32_t c1 = E.cnt1[cls];
    const unsigned long long v0 = E.vals0[cls];
    const uint32_t v1 = E.vals1[cls];
    uint32_t L0 = odd ? 24u : 24u - k, L1 = odd ? 0u : k;
#pragma unroll
    for (int i = 0; i < 24; i++) {
        const uint32_t v = (a[i >> 2] >> (8 * (i & 3))) & 0xFFu;
        if (mask1 >> i & 1u) {
            const uint32_t g = (uint32_t)__popc(__vcmpltu4(v1, v * 0x01010101u) & 0x01010101u);
            uint32_t below, at;
            cum_and_count8(c1, g, below, at);
            rk1 += exact_div_small(M1 * below, L1, E.mL);
            M1 = exact_div_small(M1 * at, L1, E.mL);
            c1 -= 1u << (8u * g);
            L1--;
        } else {
            const uint32_t g = count_below8(v0, v);
            uint32_t below, at;
            cum_and_count8(c0, g, below, at);
            rk0 += exact_div_small(M0 * below, L0, E.mL);
            M0 = exact_div_small(M0 * at, L0, E.mL);
            c0 -= 1ull << (8u * g);
            L0--;
        }
    }
    const unsigned long long p = rk1 + E.P1[cls] * rk0;          // I'' = p_S + P_S p_C
    const unsigned long long I = E.start[cls] + (unsigned long long)r +
                                 (unsigned long long)A * ((unsigned long long)s + (p << B));
    if (I >= npoints) return false;
    index = I;
    return true;
}

}  // namespace llvq
