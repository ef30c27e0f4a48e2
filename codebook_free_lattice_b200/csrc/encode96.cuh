// encode96.cuh -- the inverse map for the 96-bit budget (shells 2..214, 304,649,365 classes): a
// Leech lattice point (int8 [24]) to its packed index, one thread per vector.
//
// "Leech Lattice Vector Quantization for Efficient LLM Compression", papernotes.org notes,
// 方法详解 / 关键设计 2 (the index hierarchy, both directions).  As the 72-bit encoder
// (encode72.cuh), with:
//   - the unary class key over the coset's 30 (even: 0, 2, .., 58) or 29 (odd: 1, .., 57)
//     magnitudes: 54 or 53 bits, one u64 per class (2.4 GB, built on the device from the class
//     records); a binary search of the (shell, coset) range;
//   - the decoder's class records (start, meta, groups: off-codeword groups first, then the
//     codeword groups; odd: all groups);
//   - arrangement counts up to 24! < 2^80: the ranks in exact 128-bit arithmetic (products by
//     counts <= 24, exact divisions by L <= 24 in 64/32-bit limbs).
// A vector that is not a coded point gets the index 2^96 - 1 and raises LLVQ_FLAG_NOT_CODED.
#pragma once
#include "codec96.cuh"
#include "encode72.cuh"

namespace llvq {

constexpr int kEncShells96 = 216;

struct alignas(16) EncSmem96 {
    uint32_t golay_mask[4096];                    // ascending mask
    unsigned long long mL[32];                    // ceil(2^64 / L), L = 2..24
    uint32_t binom[25][25];                       // C(n, c)
    uint32_t seg_first[kEncShells96][2];          // classes of (shell, coset): first index
    uint32_t seg_count[kEncShells96][2];          //                            and count
    uint16_t wrank[4096];                         // codeword with top 12 bits t: place within its weight
    uint16_t nwords[32];                          // codewords of weight k
};
static_assert(sizeof(EncSmem96) % 16 == 0, "16-byte table image");

struct u128p {
    unsigned long long lo, hi;
};

__device__ __forceinline__ u128p mul_small(u128p x, uint32_t c) {
    u128p r;
    r.lo = x.lo * c;
    r.hi = x.hi * c + __umul64hi(x.lo, c);
    return r;
}

__device__ __forceinline__ u128p add128(u128p a, u128p b) {
    u128p r;
    r.lo = a.lo + b.lo;
    r.hi = a.hi + b.hi + (r.lo < a.lo ? 1ull : 0ull);
    return r;
}

// x / L for 1 <= L <= 24 (the quotient; exact when L divides x): the high word by a multiply-high
// with one correction, the low word in two 32-bit limbs
__device__ __forceinline__ u128p div_small(u128p x, uint32_t L, const unsigned long long *mL) {
    if (L == 1u) return x;
    unsigned long long qh = __umul64hi(x.hi, mL[L]);
    if (qh * L > x.hi) qh--;                                   // the estimate is q or q + 1
    uint32_t rem = (uint32_t)(x.hi - qh * L);
    const unsigned long long m = mL[L];
    const uint32_t q1 = divlimb(rem, (uint32_t)(x.lo >> 32), L, m);
    const uint32_t q0 = divlimb(rem, (uint32_t)x.lo, L, m);
    u128p q;
    q.hi = qh;
    q.lo = (unsigned long long)q1 << 32 | q0;
    return q;
}

// unary count code of the magnitudes of one coset, largest magnitude first (30 bins)
__device__ __forceinline__ unsigned long long unary_key30(const uint32_t a[6], bool odd) {
    unsigned long long h0 = 0, h1 = 0, h2 = 0;            // 5-bit counts of bins 0..11, 12..23, 24..29
#pragma unroll
    for (int i = 0; i < 24; i++) {
        const uint32_t b = ((a[i >> 2] >> (8 * (i & 3))) & 0xFFu) >> 1;
        if (b < 12u) h0 += 1ull << (5u * b);
        else if (b < 24u) h1 += 1ull << (5u * (b - 12u));
        else h2 += 1ull << (5u * (b - 24u));
    }
    unsigned long long key = 0;
#pragma unroll
    for (int b = 29; b >= 0; b--) {
        if (odd && b == 29) continue;                      // the odd coset stops at 57
        const unsigned long long h = b >= 24 ? h2 >> (5 * (b - 24)) : (b >= 12 ? h1 >> (5 * (b - 12)) : h0 >> (5 * b));
        const uint32_t c = (uint32_t)(h & 31ull);
        key = (key << (c + 1u)) | (((1ull << c) - 1ull) << 1);
    }
    return key;
}

__device__ __forceinline__ bool encode96(const uint32_t xw[6], const EncSmem96 &E, const Rec96 *__restrict__ recs,
                                         const unsigned long long *__restrict__ keys, unsigned long long np_lo,
                                         unsigned long long np_hi, unsigned long long &out_lo,
                                         unsigned long long &out_hi) {
    out_lo = ~0ull;
    out_hi = 0xFFFFFFFFull;
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
    ok &= (norm & 15) == 0 && m >= 2 && m < kEncShells96 && ((sum & 7) == (odd ? 4 : 0)) && amax <= 58u;
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
    const unsigned long long key = unary_key30(a, odd);
    const long long first = E.seg_first[m][odd], cnt = E.seg_count[m][odd];
    if (cnt == 0) return false;
    long long l = first, h = first + cnt - 1;
    while (l < h) {
        const long long mid = (l + h) >> 1;
        if (__ldg(keys + mid) < key) l = mid + 1; else h = mid;
    }
    if (__ldg(keys + l) != key) return false;
    const ulonglong2 *rp = reinterpret_cast<const ulonglong2 *>(recs + l);
    const ulonglong2 r0 = __ldg(rp);
    const uint4 cumv = __ldg(reinterpret_cast<const uint4 *>(rp + 2));
    const uint4 valv = __ldg(reinterpret_cast<const uint4 *>(rp + 3));
    const uint32_t meta = (uint32_t)(r0.y >> 32);
    const uint32_t k = (meta >> 15) & 0x1Fu, B = (meta >> 20) & 0x1Fu;
    const uint32_t A = odd ? 4096u : E.nwords[k];
    // r
    const uint32_t t12 = word >> 12;
    if (E.golay_mask[t12] != word || (!odd && (uint32_t)__popc(word) != k)) return false;
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
    // group counts: bytes of (cumulative - 0x7F) differences, 16 groups in four words
    const uint32_t cw[4] = {cumv.x, cumv.y, cumv.z, cumv.w};
    const uint32_t vw[4] = {valv.x, valv.y, valv.z, valv.w};
    uint32_t cnt16[4];
    uint32_t prev = 0;
    const uint32_t nC = odd ? 24u : 24u - k;
#pragma unroll
    for (int q = 0; q < 4; q++) {
        uint32_t wq = 0;
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const uint32_t c = ((cw[q] >> (8 * e)) & 0xFFu) - 0x7Fu;
            wq |= (c - prev) << (8 * e);
            prev = c;
        }
        cnt16[q] = wq;
    }
    // arrangements of each set: the off-S groups sum to nC counts, the rest lie on S
    u128p MC = {1ull, 0ull}, MS = {1ull, 0ull};
    uint32_t leftC = nC, leftS = 24u - nC, sumC = 0;
#pragma unroll
    for (int g = 0; g < 16; g++) {
        const uint32_t c = (cnt16[g >> 2] >> (8 * (g & 3))) & 0xFFu;
        if (c == 0u) continue;
        if (sumC < nC) { MC = mul_small(MC, E.binom[leftC][c]); leftC -= c; sumC += c; }
        else { MS = mul_small(MS, E.binom[leftS][c]); leftS -= c; }
    }
    const u128p PS = MS;
    u128p rkC = {0ull, 0ull}, rkS = {0ull, 0ull};
    uint32_t LC = nC, LS = 24u - nC;
#pragma unroll
    for (int i = 0; i < 24; i++) {
        const uint32_t v = (a[i >> 2] >> (8 * (i & 3))) & 0xFFu;
        // group: the first byte of the value list equal to v
        uint32_t G = 16u;
#pragma unroll
        for (int q = 3; q >= 0; q--) {
            const uint32_t e = __vcmpeq4(vw[q], v * 0x01010101u);
            if (e) G = 4u * q + ((uint32_t)(__ffs((int)e) - 1) >> 3);
        }
        G = min(G, 15u);
        // remaining counts of the groups before G
        uint32_t prefix = 0;
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const uint32_t lim = G > 4u * q ? min(G - 4u * q, 4u) : 0u;
            const uint32_t keep = lim >= 4u ? 0xFFFFFFFFu : ((1u << (8u * lim)) - 1u);
            prefix = (uint32_t)__dp4a(cnt16[q] & keep, 0x01010101u, prefix);
        }
        const uint32_t at = (cnt16[G >> 2] >> (8u * (G & 3u))) & 0xFFu;
        const bool onS = !odd && ((word >> i) & 1u);
        if (onS) {
            const uint32_t below = prefix - LC;              // the off-S groups come first
            rkS = add128(rkS, div_small(mul_small(MS, below), LS, E.mL));
            MS = div_small(mul_small(MS, at), LS, E.mL);
            LS--;
        } else {
            rkC = add128(rkC, div_small(mul_small(MC, prefix), LC, E.mL));
            MC = div_small(mul_small(MC, at), LC, E.mL);
            LC--;
        }
        cnt16[G >> 2] -= 1u << (8u * (G & 3u));
    }
    // I'' = p_S + P_S p_C (P_S < 2^45 when p_C != 0: either k <= 16 or the off-S set is empty)
    u128p p = rkS;
    if (rkC.lo | rkC.hi) {
        const u128p t = {PS.lo * rkC.lo, __umul64hi(PS.lo, rkC.lo) + PS.lo * rkC.hi};
        p = add128(p, t);
    }
    // t = p 2^B + s, then I = start + r + A t (all below 2^96)
    u128p t;
    t.hi = B ? (p.hi << B) | (p.lo >> (64 - B)) : p.hi;
    t.lo = (p.lo << B) | s;
    const u128p At = {t.lo * A, t.hi * A + __umul64hi(t.lo, A)};
    u128p I = {r0.x, (unsigned long long)(uint32_t)r0.y};
    I = add128(I, u128p{(unsigned long long)r, 0ull});
    I = add128(I, At);
    if (I.hi > np_hi || (I.hi == np_hi && I.lo >= np_lo)) return false;
    out_lo = I.lo;
    out_hi = I.hi;
    return true;
}

}  // namespace llvq
