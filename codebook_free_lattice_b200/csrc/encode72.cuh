// encode72.cuh -- the inverse map for the 72-bit budget (shells 2..53, 114,976 classes): a Leech
// lattice point (int8 [24]) to its packed index, one thread per vector.
//
// "Leech Lattice Vector Quantization for Efficient LLM Compression", papernotes.org notes,
// 方法详解 / 关键设计 2 (the index hierarchy, both directions).  Same steps as the 48-bit encoder
// (encode48.cuh), with the class found in global memory and 128-bit indices:
//   - class key: the magnitude multiset as a unary code read from the largest magnitude down
//     ("count ones, then a zero" for each of the 15 magnitudes of the coset, 39 bits).  Comparing
//     two descending magnitude tuples lexicographically is comparing these codes as numbers, so
//     the classes of one (shell, coset) ascend by key: a binary search of the key array;
//   - the class record is the decoder's (start, A, B, groups in decode order: codeword groups
//     ascending, then the others; odd: all groups);
//   - arrangement counts stay below 2^50.3, so the ranks use exact 64-bit integers.
// A vector that is not a coded point gets the index 2^72 - 1 and raises LLVQ_FLAG_NOT_CODED.
#pragma once
#include "codec72.cuh"
#include "encode48.cuh"

namespace llvq {

constexpr int kEncShells72 = 64;

struct alignas(16) EncSmem72 {
    uint32_t golay_mask[4096];                    // ascending mask
    unsigned long long mL[32];                    // ceil(2^64 / L), L = 2..24
    uint32_t binom[25][25];                       // C(n, c)
    uint32_t seg_first[kEncShells72][2];          // classes of (shell, coset): first index
    uint32_t seg_count[kEncShells72][2];          //                            and count
    uint16_t wrank[4096];                         // codeword with top 12 bits t: place within its weight
};
static_assert(sizeof(EncSmem72) % 16 == 0, "16-byte table image");

// unary count code of the magnitudes of one coset, largest magnitude first: 15 magnitudes
// (0, 2, .., 28 or 1, 3, .., 29), each as (count ones, one zero)
__device__ __forceinline__ unsigned long long unary_key15(const uint32_t a[6]) {
    unsigned long long hlo = 0, hhi = 0;               // 5-bit counts of bins 0..11 / 12..14
#pragma unroll
    for (int i = 0; i < 24; i++) {
        const uint32_t b = ((a[i >> 2] >> (8 * (i & 3))) & 0xFFu) >> 1;
        if (b < 12u) hlo += 1ull << (5u * b);
        else hhi += 1ull << (5u * (b - 12u));
    }
    unsigned long long key = 0;
#pragma unroll
    for (int b = 14; b >= 0; b--) {
        const uint32_t c = (uint32_t)(((b >= 12 ? hhi >> (5 * (b - 12)) : hlo >> (5 * b))) & 31ull);
        key = (key << (c + 1u)) | (((1ull << c) - 1ull) << 1);
    }
    return key;
}

// index = 2^72 - 1 marks a vector that is not coded
__device__ __forceinline__ bool encode72(const uint32_t xw[6], const EncSmem72 &E, const Rec72 *__restrict__ recs,
                                         const unsigned long long *__restrict__ keys, unsigned long long np_lo,
                                         unsigned long long np_hi, unsigned long long &lo, unsigned long long &hi) {
    lo = ~0ull;
    hi = 0xFFull;
    uint32_t a[6];
    int norm = 0, sum = 0;
    const bool odd = xw[0] & 1u;
    bool ok = true;
    uint32_t amax = 0;
#pragma unroll
    for (int q = 0; q < 6; q++) {
        a[q] = __vabsss4(xw[q]);
        ok &= (xw[q] & 0x01010101u) == (odd ? 0x01010101u : 0u);
        norm = __dp4a((int)a[q], (int)a[q], norm);
        sum = __dp4a((int)xw[q], 0x01010101, sum);
        amax = __vmaxu4(amax, a[q]);
    }
    amax = max(max(amax & 0xFFu, (amax >> 8) & 0xFFu), max((amax >> 16) & 0xFFu, amax >> 24));
    const int m = norm >> 4;
    ok &= (norm & 15) == 0 && m >= 2 && m < kEncShells72 && ((sum & 7) == (odd ? 4 : 0)) && amax <= 29u;
    uint32_t word = 0, nz = 0, neg = 0;
#pragma unroll
    for (int q = 0; q < 6; q++) {
        const uint32_t w = odd ? __vcmpeq4(xw[q] & 0x03030303u, 0x01010101u)
                               : __vcmpeq4(a[q] & 0x03030303u, 0x02020202u);
        word |= bytes_to_nibble(w) << (4 * q);
        nz |= bytes_to_nibble(__vcmpne4(a[q], 0u)) << (4 * q);
        neg |= bytes_to_nibble((xw[q] >> 7) & 0x01010101u) << (4 * q);
    }
    if (!ok) return false;
    // class: binary search of the (shell, coset) keys
    const unsigned long long key = unary_key15(a);
    const int first = (int)E.seg_first[m][odd], cnt = (int)E.seg_count[m][odd];
    if (cnt == 0) return false;
    int l = first, h = first + cnt - 1;
    while (l < h) {
        const int mid = (l + h) >> 1;
        if (__ldg(keys + mid) < key) l = mid + 1; else h = mid;
    }
    if (__ldg(keys + l) != key) return false;
    const Rec72 &R = recs[l];
    const unsigned long long st_lo = R.start_lo, st_hi = R.start_hi;
    const uint32_t A = R.A, B = R.B, nS = R.nS;
    const unsigned long long cum = R.cum, vals = R.vals;
    const uint32_t val8 = R.val8, ng = R.ngroups;
    // r
    const uint32_t t12 = word >> 12;
    if (E.golay_mask[t12] != word || (!odd && (uint32_t)__popc(word) != nS)) return false;
    const uint32_t r = odd ? t12 : E.wrank[t12];
    // s (even)
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
    // group counts (decode order: codeword groups ascending, then the others; odd: all)
    unsigned long long cnt8 = 0;                     // bytes: counts of groups 0..7
    uint32_t prev = 0;
#pragma unroll
    for (int g = 0; g < 8; g++) {
        const uint32_t c = (uint32_t)(cum >> (8 * g)) & 0xFFu;
        cnt8 |= (unsigned long long)(c - prev) << (8 * g);
        prev = c;
    }
    uint32_t c_last = ng > 8u ? 24u - prev : 0u;    // group 8
    // arrangements of each coordinate set: products of binomials over its groups
    unsigned long long MS = 1, MC = 1;
    uint32_t nleftS = odd ? 24u : nS, nleftC = odd ? 0u : 24u - nS;
#pragma unroll
    for (int g = 0; g < 9; g++) {
        const uint32_t c = g < 8 ? (uint32_t)(cnt8 >> (8 * g)) & 0xFFu : c_last;
        const uint32_t v = g < 8 ? (uint32_t)(vals >> (8 * g)) & 0xFFu : val8;
        if ((uint32_t)g >= ng) continue;
        const bool onS = odd || (v & 3u) == 2u;
        if (onS) { MS *= E.binom[nleftS][c]; nleftS -= c; }
        else { MC *= E.binom[nleftC][c]; nleftC -= c; }
    }
    const unsigned long long PS = MS;
    unsigned long long rkS = 0, rkC = 0;
    uint32_t LS = odd ? 24u : nS, LC = odd ? 0u : 24u - nS;
#pragma unroll
    for (int i = 0; i < 24; i++) {
        const uint32_t v = (a[i >> 2] >> (8 * (i & 3))) & 0xFFu;
        // group index: the byte of vals equal to v (group 8 when none)
        const uint32_t e0 = __vcmpeq4((uint32_t)vals, v * 0x01010101u), e1 = __vcmpeq4((uint32_t)(vals >> 32), v * 0x01010101u);
        const unsigned long long eq = (unsigned long long)e1 << 32 | e0;
        uint32_t G = eq ? (uint32_t)(__ffsll((long long)eq) - 1) >> 3 : 8u;
        G = min(G, ng - 1u);
        const unsigned long long keep = G >= 8u ? ~0ull : ((1ull << (8u * G)) - 1ull);
        const unsigned long long pl = cnt8 & keep;
        const uint32_t prefix = (uint32_t)__dp4a((uint32_t)pl, 0x01010101u, __dp4a((uint32_t)(pl >> 32), 0x01010101u, 0u));
        const uint32_t at = G < 8u ? (uint32_t)(cnt8 >> (8u * G)) & 0xFFu : c_last;
        const bool onS = odd || ((word >> i) & 1u);
        if (onS) {
            rkS += exact_div_small(MS * prefix, LS, E.mL);
            MS = exact_div_small(MS * at, LS, E.mL);
            LS--;
        } else {
            const uint32_t below = prefix - LS;          // the codeword groups come first
            rkC += exact_div_small(MC * below, LC, E.mL);
            MC = exact_div_small(MC * at, LC, E.mL);
            LC--;
        }
        if (G < 8u) cnt8 -= 1ull << (8u * G);
        else c_last--;
    }
    // I = start + r + A (s + 2^B I''), I'' = p_S + P_S p_C (odd: p_C = 0)
    const unsigned long long p = rkS + PS * rkC;
    const unsigned long long ph = B ? (p >> (64 - B)) : 0ull, pl2 = p << B;   // p 2^B (128-bit)
    const unsigned long long t_lo = pl2 + s, t_hi = ph + (t_lo < pl2 ? 1ull : 0ull);
    // A * t (A <= 4096, t < 2^76)
    const unsigned long long m_lo = t_lo * A, m_hi = __umul64hi(t_lo, A) + t_hi * A;
    unsigned long long r_lo = st_lo + r;
    unsigned long long r_hi = st_hi + (r_lo < st_lo ? 1ull : 0ull);
    r_lo += m_lo;
    r_hi += m_hi + (r_lo < m_lo ? 1ull : 0ull);
    if (r_hi > np_hi || (r_hi == np_hi && r_lo >= np_lo)) return false;
    lo = r_lo;
    hi = r_hi;
    return true;
}

}  // namespace llvq
