// codec72.cuh -- decoder for the 72-bit index budget (3 bits per weight: shells 2..53,
// 114,976 classes), one thread per 24-weight block.
//
// Same hierarchy as the 48-bit decoder ("Leech Lattice Vector Quantization for Efficient LLM
// Compression", papernotes.org notes, 方法详解 / 关键设计 2), with wider arithmetic:
//   - indices are 72-bit (word = two little-endian 64-bit halves; gain code in bits 72..79);
//   - class records (96 B) and the guide table on the top 16 index bits live in global memory
//     (L2-resident, 9.5 MB), the Golay tables in shared memory;
//   - I_class < 2^63, so r, s, I'' come from one 64-bit division by A (a multiply-high by a
//     per-class reciprocal and one correction);
//   - arrangement counts reach P ~ 2^50.2, beyond fp64, so the arithmetic decoding state is
//     a 64-bit fixed-point fraction kept above the exact value: slot = high word of phi * L,
//     and phi <- (slot_in_group * 2^64 + low word) * R_c with R_c = ceil(2^64 / c) (plus one).
//     An even class ranks S and the other positions separately (I'' = p_S + P_S p_C):
//     phi_C ~ 2^64 I''/P decodes the positions off S and phi_S = phi_C * P_C mod 2^64
//     ~ 2^64 p_S/P_S decodes S.  Each step adds at most c + 1 units of error, the start
//     error of phi_S is below 2 P_C units, and 24 * 577 * P <= 2^64 for every class, so every
//     slot is exact (the bound argument is in the design notes);
//   - up to 9 magnitude groups: cumulative counts in 8 bytes; group 8 patched in when present.
#pragma once
#include "device_common.cuh"

namespace llvq {

struct alignas(16) Rec72 {
    unsigned long long start_lo, start_hi;   // first global index of the class (128-bit)
    unsigned long long Rint, Rfrac;          // 2^64 / P: integer part, fraction * 2^64 (up)
    unsigned long long cum;                  // bytes: C_<=g, g = 0..7 (saturating at 24)
    unsigned long long vals;                 // bytes: magnitudes of groups 0..7
    uint32_t flo, fhi;                       // bytes: per-group sign flags, groups 0..7
    uint32_t A;                              // 1, 759, 2576 or 4096
    uint8_t val8, flag8;                     // magnitude / sign flag of group 8
    uint8_t nS, B, flags, m, ngroups, pad0;  // flags: bit0 odd coset, bit1 parity target
    uint16_t wbase, pad1;
    uint32_t pad2;
    unsigned long long PC;                   // arrangements off S (even), 1 for odd classes
    unsigned long long mA;                   // floor((2^64 - 1) / A): I_class / A by multiply-high
};
static_assert(sizeof(Rec72) == 96, "Rec72 layout");

constexpr int kGuideBits72 = 16;                  // 65536 buckets over [0, 2^72)

struct alignas(16) Smem72 {
    uint32_t golay_mask[4096];
    uint32_t golay_weight[4096];
    unsigned long long rc[32];                    // ceil(2^64 / c), c = 2..24 (0 for c <= 1)
    uint16_t pdep_off[256];
    uint8_t pdep[kPdepEntries];
    float invnorm[64];                            // 1 / (4 sqrt(m)), m <= 53
};

static_assert(sizeof(Smem72) % 16 == 0, "16-byte table image");

struct Dec72 {
    using Word = ulonglong2;                      // x = bits 0..63, y = bits 64..127
    using Smem = Smem72;
    struct Args {
        const Smem72 *image;
        const Rec72 *recs;
        const uint32_t *guide;                    // [2^16 + 1] class index per bucket
        unsigned long long np_lo, np_hi;          // N_M
    };
    static constexpr int kWordBytes = 16;
    static constexpr int kCtasPerSm = 2;

    __device__ static Word load(const Word *p) { return __ldg(p); }
    __device__ static int gain_code(const Word &w) { return (int)((w.y >> 8) & 0xFFu); }
    __device__ static float invnorm(const Smem &S, int m) { return S.invnorm[m]; }

    __device__ static bool decode(const Word &w, const Smem &S, const Args &a, uint32_t v[6], int &m) {
        unsigned long long lo = w.x, hi = w.y & 0xFFull;
        const bool ok = hi < a.np_hi || (hi == a.np_hi && lo < a.np_lo);
        if (!ok) { lo = 0; hi = 0; }
        // 1. class: guide bucket on the top 16 bits, then binary search of the starts
        const uint32_t b = (uint32_t)((hi << 8) | (lo >> 56));
        int clo = (int)__ldg(a.guide + b), chi = (int)__ldg(a.guide + b + 1);
        while (clo < chi) {
            const int mid = (clo + chi + 1) >> 1;
            const ulonglong2 st = __ldg(reinterpret_cast<const ulonglong2 *>(a.recs + mid));
            const bool le = st.y < hi || (st.y == hi && st.x <= lo);
            if (le) clo = mid; else chi = mid - 1;
        }
        const Rec72 R = a.recs[clo];
        m = R.m;
        // 2. I_class = idx - start < 2^63 (the high halves cancel), then r, s, I''
        const unsigned long long Ic = lo - R.start_lo;
        // q = floor(I_class / A): the multiply-high by floor((2^64 - 1)/A) is q or q - 1
        unsigned long long q = __umul64hi(Ic, R.mA);
        uint32_t r = (uint32_t)(Ic - q * R.A);
        if (r >= R.A) { q += 1; r -= R.A; }
        const uint32_t s = (uint32_t)(q & ((1ull << R.B) - 1ull));
        const unsigned long long p = q >> R.B;
        // 3. codeword
        const bool odd = R.flags & 1u;
        const uint32_t word = odd ? S.golay_mask[r & 4095u] : S.golay_weight[min(R.wbase + r, 4095u)];
        const uint32_t side0 = odd ? 0xFFFFFFu : word;
        // 4. arrangement in 64-bit fixed point
        unsigned long long phiC = p * R.Rint + __umul64hi(p, R.Rfrac) + 1ull;   // off S
        unsigned long long phiS = phiC * R.PC;                                    // on S
        uint32_t clo4 = (uint32_t)R.cum + 0x7F7F7F7Fu, chi4 = (uint32_t)(R.cum >> 32) + 0x7F7F7F7Fu;
        int L0 = R.nS, L1 = 24 - R.nS;
        uint32_t sel[6] = {0, 0, 0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < 24; i++) {
            const bool on0 = side0 & (1u << i);
            const uint32_t L = (uint32_t)(on0 ? L0 : L1);
            const uint32_t off = on0 ? 0u : (uint32_t)L0;
            const unsigned long long phi = on0 ? phiS : phiC;
            const unsigned long long frac = phi * L;
            const uint32_t slot = (uint32_t)__umul64hi(phi, L) + off;
            const uint32_t ulo = clo4 - slot * 0x01010101u, uhi = chi4 - slot * 0x01010101u;
            const uint32_t dlo = (ulo >> 7) & 0x01010101u, dhi = (uhi >> 7) & 0x01010101u;
            const uint32_t grp = 8u - (uint32_t)__dp4a((int)dlo, 0x01010101, __dp4a((int)dhi, 0x01010101, 0));
            const uint32_t stb = __byte_perm(clo4, chi4, (grp - 1u) & 7u) & 0xFFu;
            const uint32_t enb = __byte_perm(clo4, chi4, grp & 7u) & 0xFFu;
            const uint32_t st = grp ? stb - 0x7Fu : 0u;                        // C_<grp
            const uint32_t en = grp < 8u ? enb - 0x7Fu : (uint32_t)(24 - i);  // C_<=grp
            const uint32_t cnt = min(en - st, 31u);                            // in 1..24
            const unsigned long long rc = S.rc[cnt];
            const unsigned long long within = slot - st;                       // < cnt
            const unsigned long long phn = cnt == 1u ? frac + 1ull : within * rc + __umul64hi(frac, rc) + 1ull;
            if (on0) phiS = phn; else phiC = phn;
            clo4 -= dlo;
            chi4 -= dhi;
            L0 -= on0 ? 1 : 0;
            L1 -= on0 ? 0 : 1;
            sel[i >> 2] |= grp << (4 * (i & 3));
        }
        // 5. magnitudes, sign flags (group 8 patched in when the class has nine groups), signs
        const uint32_t vlo = (uint32_t)R.vals, vhi = (uint32_t)(R.vals >> 32);
        uint32_t mag[6], F = 0;
#pragma unroll
        for (int q2 = 0; q2 < 6; q2++) {
            const uint32_t s7 = sel[q2] & 0x7777u;
            mag[q2] = __byte_perm(vlo, vhi, s7);
            uint32_t fb = __byte_perm(R.flo, R.fhi, s7);
            if (R.ngroups > 8) {
                const uint32_t h = (sel[q2] >> 3) & 0x1111u;          // nibbles holding group 8
                const uint32_t nib = (h & 1u) | ((h >> 3) & 2u) | ((h >> 6) & 4u) | ((h >> 9) & 8u);
                const uint32_t mb = nibble_to_bytes(nib) * 0xFFu;
                mag[q2] = (mag[q2] & ~mb) | ((uint32_t)R.val8 * 0x01010101u & mb);
                fb = (fb & ~mb) | ((uint32_t)R.flag8 * 0x01010101u & mb);
            }
            F |= bytes_to_nibble(fb) << (4 * q2);
        }
        apply_signs(odd, word, s, F, (uint32_t)(R.flags >> 1), mag, ok, S.pdep_off, S.pdep, v);
        return ok;
    }
};

}  // namespace llvq
