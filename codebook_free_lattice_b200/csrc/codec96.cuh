// codec96.cuh -- decoder for the 96-bit index budget (4 bits per weight: shells 2..214,
// 304,649,365 classes), one thread per 24-weight block.
//
// Same hierarchy as the 48- and 72-bit decoders ("Leech Lattice Vector Quantization for
// Efficient LLM Compression", papernotes.org notes, 方法详解 / 关键设计 2), with the class table
// in global memory and 128-bit arithmetic:
//   - class: a guide on the top 28 index bits gives the range of class records that can hold the
//     index (usually one to three), then a binary search of their starts;
//   - I_class = I - start < 2^92; r = I_class mod A and q = I_class / A by long division in
//     32-bit limbs (a multiply-high by ceil(2^64 / A) per limb is exact for numerators < A 2^32);
//     s = q mod 2^B, p = q / 2^B;
//   - arrangement counts reach P ~ 2^79, so the arithmetic-decoding state is a 128-bit
//     fixed-point fraction phi >= 2^128 p / P, started from the class's stored reciprocal
//     R = ceil(2^(128+t) / P) (t = bitlen(P - 1)) as phi = floor(p R / 2^t) + 1.  A step takes
//     slot = high word of phi * L and, for the group a holding the slot,
//     phi <- floor(((slot - C_<a) 2^128 + low words) / c_a) + 1 by long division in 32-bit limbs.
//     With e_i = (phi_i - 2^128 f_i) P_i / 2^128 (P_i = arrangements left), e_{i+1} <= e_i +
//     P_{i+1} / 2^128, so e stays below 2^-40 over the 24 steps and every slot is exact.
//     Once every lane of the warp has P_i < 2^57 (a running upper bound on log2 P_i), the state
//     narrows to its top 64 bits plus one and the steps continue in two limbs: the same bound in
//     units of 2^-64 gives e <= 2^-7 + 24 * 2^-7 < 1.  The last step needs no new state;
//   - an even class ranks its magnitudes off and on the codeword separately with
//     I'' = p_S + P_S p_C, which is the lexicographic rank of the concatenated sequence
//     (positions off S ascending, then positions on S ascending): one state walks the positions
//     off S first, then those on S, over one list of magnitude groups (off-S groups, then on-S
//     groups) whose cumulative counts sit in 16 bytes.
#pragma once
#include "device_common.cuh"
#include "tables96.h"

namespace llvq {

constexpr int kGuideShift96 = 68;                 // guide bucket = index >> 68 (top 28 bits)

struct alignas(16) Smem96 {
    uint32_t golay_mask[4096];
    uint32_t golay_weight[4096];
    unsigned long long mc[32];                    // ceil(2^64 / c), c = 2..24 (0 for c <= 1)
    unsigned long long mA[32];                    // ceil(2^64 / A) for A = codewords of weight k (k <= 24), [25]: A = 4096
    uint16_t nwords[32];                          // A: codewords of weight k, [25] = 4096
    uint16_t wbase[32];                           // first by-weight slot of weight k
    float lg2_down[32];                           // log2(L) rounded down, L = 1..24
    float lg2_up[32];                             // log2(c) rounded up, c = 1..24
    uint16_t pdep_off[256];
    uint8_t pdep[kPdepEntries];
    float invnorm[256];                           // 1 / (4 sqrt(m)), m <= 214
};
static_assert(sizeof(Smem96) % 16 == 0, "16-byte table image");

constexpr float kNarrowLog2_96 = 57.0f;           // 64-bit state once every lane has P_i < 2^57

// 64 x 64 -> 128-bit product
__device__ __forceinline__ void mul64wide(unsigned long long a, unsigned long long b, unsigned long long &lo,
                                          unsigned long long &hi) {
    lo = a * b;
    hi = __umul64hi(a, b);
}

// one limb of a long division by a small divisor d (rem < d): (rem 2^32 + x) / d through the
// multiply-high by m = ceil(2^64 / d), exact for numerators below d 2^32 and d <= 4096
__device__ __forceinline__ uint32_t divlimb(uint32_t &rem, uint32_t x, uint32_t d, unsigned long long m) {
    const unsigned long long num = (unsigned long long)rem << 32 | x;
    const uint32_t q = d == 1u ? x : (uint32_t)__umul64hi(num, m);
    rem = x - q * d;
    return q;
}

// byte j (0..15) of the 16 bytes y0..y3
__device__ __forceinline__ uint32_t byte16(uint32_t y0, uint32_t y1, uint32_t y2, uint32_t y3, uint32_t j) {
    const uint32_t lo = __byte_perm(y0, y1, j & 7u), hi = __byte_perm(y2, y3, j & 7u);
    return ((j & 8u) ? hi : lo) & 0xFFu;
}

struct Dec96 {
    using Word = ulonglong2;                      // x = bits 0..63, y = bits 64..127
    using Smem = Smem96;
    struct Args {
        const Smem96 *image;
        const Rec96 *recs;
        const uint32_t *guide;                    // class index per bucket of the top 28 index bits
        unsigned long long np_lo;                 // N_M, bits 0..63
        uint32_t np_hi;                           // N_M, bits 64..95
    };
    static constexpr int kWordBytes = 16;
    static constexpr int kCtasPerSm = 2;

    __device__ static Word load(const Word *p) { return __ldg(p); }
    __device__ static int gain_code(const Word &w) { return (int)((w.y >> 32) & 0xFFu); }
    __device__ static float invnorm(const Smem &S, int m) { return S.invnorm[m]; }

    __device__ static bool decode(const Word &w, const Smem &S, const Args &a, uint32_t v[6], int &m) {
        unsigned long long lo = w.x;
        uint32_t hi = (uint32_t)w.y;
        const bool ok = hi < a.np_hi || (hi == a.np_hi && lo < a.np_lo);
        if (!ok) { lo = 0; hi = 0; }
        // 1. class: guide bucket on the top 28 bits, then binary search of the starts
        const uint32_t b = hi >> (kGuideShift96 - 64);
        int clo = (int)__ldg(a.guide + b), chi = (int)__ldg(a.guide + b + 1);
        while (clo < chi) {
            const int mid = (clo + chi + 1) >> 1;
            const ulonglong2 st = __ldg(reinterpret_cast<const ulonglong2 *>(a.recs + mid));
            const uint32_t sh = (uint32_t)st.y;
            const bool le = sh < hi || (sh == hi && st.x <= lo);
            if (le) clo = mid; else chi = mid - 1;
        }
        const ulonglong2 *rp = reinterpret_cast<const ulonglong2 *>(a.recs + clo);
        const ulonglong2 r0 = __ldg(rp), r1 = __ldg(rp + 1);
        const uint4 cumv = __ldg(reinterpret_cast<const uint4 *>(rp + 2));
        const uint4 valv = __ldg(reinterpret_cast<const uint4 *>(rp + 3));
        const uint32_t meta = (uint32_t)(r0.y >> 32);
        m = (int)((meta >> 7) & 0xFFu);
        const bool odd = meta & kMeta96Odd;
        const uint32_t k = (meta >> 15) & 0x1Fu, B = (meta >> 20) & 0x1Fu;
        const int t = (int)(meta & 0x7Fu);
        // 2. I_class = I - start < 2^92; r = I_class mod A, q = I_class / A (three 32-bit limbs)
        const unsigned long long clo64 = lo - r0.x;
        const uint32_t chi32 = hi - (uint32_t)r0.y - (lo < r0.x ? 1u : 0u);
        const uint32_t A = odd ? 4096u : S.nwords[k];
        const unsigned long long mAk = S.mA[odd ? 25u : k];
        uint32_t r = 0;
        const uint32_t q2 = divlimb(r, chi32, A, mAk);
        const uint32_t q1 = divlimb(r, (uint32_t)(clo64 >> 32), A, mAk);
        const uint32_t q0 = divlimb(r, (uint32_t)clo64, A, mAk);
        const unsigned long long qlo = (unsigned long long)q1 << 32 | q0;
        const uint32_t s = (uint32_t)(qlo & ((1ull << B) - 1ull));
        const unsigned long long plo = B ? (qlo >> B) | ((unsigned long long)q2 << (64 - B)) : qlo;
        const unsigned long long phig = (unsigned long long)(q2 >> B);   // p, bits 64..79
        // 3. codeword: S (even, by weight) or T (odd, by mask)
        const uint32_t word = odd ? S.golay_mask[r & 4095u] : S.golay_weight[min((uint32_t)S.wbase[k] + r, 4095u)];
        // 4. phi = p' + hi128(p' R') + 1 with p' = p 2^(128 - t) (p < P <= 2^t)
        unsigned long long F0 = 1ull, F1 = 0ull;
        if (t > 0) {
            const int u = 128 - t;                                     // 48..127
            unsigned long long P0, P1;
            if (u >= 64) { P1 = plo << (u - 64); P0 = 0ull; }
            else { P1 = (phig << u) | (plo >> (64 - u)); P0 = plo << u; }
            const unsigned long long R0 = r1.x, R1 = r1.y;
            unsigned long long a0l, a0h, a1l, a1h, b0l, b0h, b1l, b1h;
            mul64wide(P0, R0, a0l, a0h);
            mul64wide(P0, R1, a1l, a1h);
            mul64wide(P1, R0, b0l, b0h);
            mul64wide(P1, R1, b1l, b1h);
            // middle word: a0h + a1l + b0l; its carries go into the high 128 bits
            unsigned long long mid = a0h + a1l;
            unsigned long long cy = mid < a0h ? 1ull : 0ull;
            mid += b0l;
            cy += mid < b0l ? 1ull : 0ull;
            // high 128 bits: b1 + a1h + b0h + cy
            unsigned long long h0 = b1l + a1h;
            unsigned long long h1 = b1h + (h0 < a1h ? 1ull : 0ull);
            h0 += b0h;
            h1 += h0 < b0h ? 1ull : 0ull;
            h0 += cy;
            h1 += h0 < cy ? 1ull : 0ull;
            // phi = p' + high + 1
            F0 = P0 + h0;
            F1 = P1 + h1 + (F0 < P0 ? 1ull : 0ull);
            F0 += 1ull;
            F1 += F0 == 0ull ? 1ull : 0ull;
            (void)a0l;
        }
        uint32_t f0 = (uint32_t)F0, f1 = (uint32_t)(F0 >> 32), f2 = (uint32_t)F1, f3 = (uint32_t)(F1 >> 32);
        // 5. 24 steps: positions off the codeword (ascending), then on it; odd: all, ascending
        uint32_t y0 = cumv.x, y1 = cumv.y, y2 = cumv.z, y3 = cumv.w;
        const uint32_t nC = odd ? 24u : 24u - k;
        uint32_t cm = odd ? 0xFFFFFFu : (~word & 0xFFFFFFu), sm = word;
        uint32_t sel0 = 0, sel1 = 0, sel2 = 0;
        float lp = (float)t;                                             // >= log2 P_i
        bool wide = true;
#pragma unroll
        for (int i = 0; i < 24; i++) {
            const bool inC = (uint32_t)i < nC;
            const uint32_t L = inC ? nC - (uint32_t)i : 24u - (uint32_t)i;
            if (wide && !__any_sync(__activemask(), lp >= kNarrowLog2_96)) {
                // narrow to the top 64 bits plus one (uniform over the lanes that vote together;
                // a lane narrows only when its own bound is below the threshold)
                const unsigned long long h = ((unsigned long long)f3 << 32 | f2) + 1ull;
                f2 = (uint32_t)h;
                f3 = (uint32_t)(h >> 32);
                wide = false;
            }
            // phi * L: the fraction (low limbs) and the slot above it
            unsigned long long t0 = 0, t1 = 0, t2, t3;
            if (wide) {
                t0 = (unsigned long long)f0 * L;
                t1 = (unsigned long long)f1 * L + (t0 >> 32);
                t2 = (unsigned long long)f2 * L + (t1 >> 32);
            } else {
                t2 = (unsigned long long)f2 * L;
            }
            t3 = (unsigned long long)f3 * L + (t2 >> 32);
            const uint32_t slot = (uint32_t)(t3 >> 32);
            // group: the number of cumulative counts C_<=g at or below the slot
            const uint32_t sb = slot * 0x01010101u;
            const uint32_t d0 = ((y0 - sb) >> 7) & 0x01010101u, d1 = ((y1 - sb) >> 7) & 0x01010101u;
            const uint32_t d2 = ((y2 - sb) >> 7) & 0x01010101u, d3 = ((y3 - sb) >> 7) & 0x01010101u;
            const uint32_t above = (uint32_t)__dp4a(d0, 0x01010101u, __dp4a(d1, 0x01010101u,
                                   __dp4a(d2, 0x01010101u, __dp4a(d3, 0x01010101u, 0u))));
            const uint32_t grp = 16u - above;
            const uint32_t en = byte16(y0, y1, y2, y3, grp) - 0x7Fu;                    // C_<=grp
            const uint32_t st = grp ? byte16(y0, y1, y2, y3, grp - 1u) - 0x7Fu : 0u;   // C_<grp
            const uint32_t c = min(en - st, 31u);
            y0 -= d0;
            y1 -= d1;
            y2 -= d2;
            y3 -= d3;
            if (i < 23) {                                  // the last step needs no new state
                // phi <- floor((slot - C_<a) 2^W + fraction) / c) + 1, W = 128 or 64
                uint32_t rem = slot - st;                                  // < c
                const unsigned long long mc = S.mc[c];
                const uint32_t n3 = divlimb(rem, (uint32_t)t3, c, mc);
                const uint32_t n2 = divlimb(rem, (uint32_t)t2, c, mc);
                if (wide) {
                    const uint32_t n1 = divlimb(rem, (uint32_t)t1, c, mc);
                    const uint32_t n0 = divlimb(rem, (uint32_t)t0, c, mc);
                    const unsigned long long lo64 = ((unsigned long long)n1 << 32 | n0) + 1ull;
                    const unsigned long long hi64 = ((unsigned long long)n3 << 32 | n2) + (lo64 == 0ull ? 1ull : 0ull);
                    f0 = (uint32_t)lo64;
                    f1 = (uint32_t)(lo64 >> 32);
                    f2 = (uint32_t)hi64;
                    f3 = (uint32_t)(hi64 >> 32);
                } else {
                    const unsigned long long h64 = ((unsigned long long)n3 << 32 | n2) + 1ull;
                    f2 = (uint32_t)h64;
                    f3 = (uint32_t)(h64 >> 32);
                }
                lp = lp - S.lg2_down[L] + S.lg2_up[c];                     // P_{i+1} = P_i c / L
            }
            // coordinate of this step: the lowest position left in its set
            const uint32_t mk = inC ? cm : sm;
            const uint32_t pos = (uint32_t)__ffs((int)mk) - 1u;
            const uint32_t rest = mk & (mk - 1u);
            cm = inC ? rest : cm;
            sm = inC ? sm : rest;
            const uint32_t nib = grp << (4u * (pos & 7u));
            sel0 |= pos < 8u ? nib : 0u;
            sel1 |= (pos >= 8u && pos < 16u) ? nib : 0u;
            sel2 |= pos >= 16u ? nib : 0u;
        }
        // 6. magnitudes by group (16 bytes), sign flags (odd: |x| = 1 mod 4; even: x != 0), signs
        uint32_t mag[6], F = 0;
#pragma unroll
        for (int q = 0; q < 6; q++) {
            const uint32_t word4 = q < 2 ? sel0 : (q < 4 ? sel1 : sel2);
            const uint32_t nibs = (word4 >> (16 * (q & 1))) & 0xFFFFu;
            const uint32_t s7 = nibs & 0x7777u;
            const uint32_t mlo = __byte_perm(valv.x, valv.y, s7), mhi = __byte_perm(valv.z, valv.w, s7);
            const uint32_t h = (nibs >> 3) & 0x1111u;                   // group index bit 3
            const uint32_t nib4 = (h & 1u) | ((h >> 3) & 2u) | ((h >> 6) & 4u) | ((h >> 9) & 8u);
            const uint32_t mb = nibble_to_bytes(nib4) * 0xFFu;
            mag[q] = (mlo & ~mb) | (mhi & mb);
            const uint32_t fb = odd ? __vcmpeq4(mag[q] & 0x03030303u, 0x01010101u) : __vcmpne4(mag[q], 0u);
            F |= bytes_to_nibble(fb) << (4 * q);
        }
        apply_signs(odd, word, s, F, (meta >> 26) & 1u, mag, ok, S.pdep_off, S.pdep, v);
        return ok;
    }
};

}  // namespace llvq
