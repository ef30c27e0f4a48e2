// codec48.cuh -- decoder for the 48-bit index budget (2 bits per weight: shells 2..13,
// 383 classes), one thread per 24-weight block.
//
// Method: "Leech Lattice Vector Quantization for Efficient LLM Compression", papernotes.org
// notes, 方法详解 / 关键设计 2 (shell and class by cumulative offsets; r = I_class mod A,
// I' = floor(I_class / A), s = I' mod 2^B, I'' = floor(I' / 2^B)).
//
//   1. class: a guide table on the top index bits narrows a binary search of the class starts;
//   2. r, s, I'' by one fp64 division by A with an exact integer correction;
//   3. codeword from the shared-memory Golay tables (odd: T by mask order; even: S among the
//      codewords of weight k);
//   4. the arrangement rank I'' is unranked coordinate by coordinate as exact arithmetic
//      decoding.  An even class ranks the magnitudes on its codeword S and on the other
//      positions separately, I'' = p_S + P_S p_C, each lexicographically; an odd class has one
//      coordinate set.  f_C = I''/P (fp64, rounded upward) equals (p_C + p_S/P_S)/P_C from above
//      and decodes the positions off S; f_S = f_C P_C - p_C = p_S/P_S from above decodes S.  At a
//      coordinate whose set has L places left, the slot floor(f * L) picks the magnitude group
//      among that set's remaining items (byte-SIMD search of the cumulative counts) and
//      f <- (f * L - start(group)) / count(group).  Directed rounding keeps each f above its exact
//      rational with an error far below 1/(remaining arrangements) for P < 2^33, so every slot
//      is exact.  The loop stays on the FMA, ALU and fp64 pipes;
//   5. magnitudes and sign flags by byte permutation of the class's group tables, then signs.
#pragma once
#include "device_common.cuh"

namespace llvq {

struct alignas(16) Rec48 {
    unsigned long long start;  // first global index of the class
    double invP;               // 1/P rounded toward +inf
    double invA;               // 1/A rounded to nearest
    uint32_t cum;              // bytes: cumulative counts C_<=g, g = 0..3 (saturating at 24)
    uint32_t vals;             // bytes: magnitudes of groups 0..3
    uint32_t A;                // 1, 759, 2576 or 4096
    uint32_t gflag;            // bytes: per-group sign flag, groups 0..3 (odd: |x| = 1 mod 4;
                               //        even: |x| != 0)
    uint8_t val4;              // magnitude of group 4
    uint8_t gflag4;            // sign flag of group 4
    uint8_t nS;                // places on the codeword side: k (even) or 24 (odd)
    uint8_t B;                 // free sign bits
    uint8_t flags;             // bit0 odd coset, bit1 parity target (sum|x|/4 odd)
    uint8_t m;                 // shell
    uint16_t wbase;            // even: first by-weight Golay slot of weight k
    double PC;                 // arrangements off S (even; exact, < 2^24), 1 for odd classes
    double pad;
};
static_assert(sizeof(Rec48) == 64, "Rec48 layout");

constexpr int kGuideBits48 = 11;                  // 2048 buckets over [0, 2^48)
constexpr int kGuideShift48 = 48 - kGuideBits48;

// Shared-memory image of the 48-bit decode tables (one copy per CTA, 72 KB).
struct Smem48 {
    uint32_t golay_mask[4096];
    uint32_t golay_weight[4096];
    double invc[32];                              // 1/c rounded up, c = 1..24
    unsigned long long starts[400];               // class starts, [nclasses] = N_M
    Rec48 recs[384];
    uint16_t guide[(1 << kGuideBits48) + 1];
    uint16_t pdep_off[256];
    uint8_t pdep[kPdepEntries];
    float invnorm[16];                            // 1 / (4 sqrt(m))
};

struct Dec48 {
    using Word = unsigned long long;
    using Smem = Smem48;
    struct Args {
        const Smem48 *image;
        unsigned long long npoints;
    };
    static constexpr int kWordBytes = 8;
    static constexpr int kCtasPerSm = 3;          // 40 registers, 72 KB shared per CTA

    __device__ static Word load(const Word *p) { return __ldg(p); }
    __device__ static int gain_code(const Word &w) { return (int)((w >> 48) & 0xFFu); }
    __device__ static float invnorm(const Smem &S, int m) { return S.invnorm[m]; }

    // Decode one packed word into 24 signed int8 coordinates (v[q] byte b = coordinate 4q+b).
    // Returns false (and v = 0) for an index >= N_M.  m receives the shell.
    __device__ static bool decode(const Word &w, const Smem &S, const Args &a, uint32_t v[6], int &m) {
        unsigned long long idx = w & 0xFFFFFFFFFFFFull;
        const bool ok = idx < a.npoints;
        if (!ok) idx = 0;
        // 1. class
        int lo = S.guide[idx >> kGuideShift48];
        int hi = S.guide[(idx >> kGuideShift48) + 1];
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (S.starts[mid] <= idx) lo = mid; else hi = mid - 1;
        }
        const Rec48 R = S.recs[lo];
        m = R.m;
        // 2. I_class = r + A (s + 2^B I'')
        const unsigned long long Ic = idx - R.start;
        unsigned long long q = (unsigned long long)((double)Ic * R.invA);
        long long rem = (long long)(Ic - q * R.A);
        if (rem < 0) { q -= 1; rem += R.A; }
        else if (rem >= (long long)R.A) { q += 1; rem -= R.A; }
        const uint32_t r = (uint32_t)rem;
        const uint32_t s = (uint32_t)(q & ((1ull << R.B) - 1ull));
        const unsigned long long p = q >> R.B;
        // 3. codeword
        const bool odd = R.flags & 1u;
        const uint32_t word = odd ? S.golay_mask[r & 4095u] : S.golay_weight[min(R.wbase + r, 4095u)];
        const uint32_t side0 = odd ? 0xFFFFFFu : word;
        // 4. arrangement.  Byte b of cumB is 0x7F + C_<=b (remaining items of groups 0..b),
        //    biased one below the guard bit so the byte-wise subtraction of the slot never borrows.
        double fC = __dmul_ru((double)p, R.invP);                   // (p_C + p_S/P_S) / P_C
        const double g0 = __dmul_ru(fC, R.PC);                       // p_C + p_S/P_S
        double fS = __dadd_ru(g0, 0x1p52 - __dadd_rz(g0, 0x1p52));   // p_S / P_S
        uint32_t cumB = R.cum + 0x7F7F7F7Fu;
        int L0 = R.nS, L1 = 24 - R.nS;
        uint32_t sel[6] = {0u - 0x3333u, 0u - 0x3333u, 0u - 0x3333u,
                           0u - 0x3333u, 0u - 0x3333u, 0u - 0x3333u};
#pragma unroll
        for (int i = 0; i < 24; i++) {
            const bool on0 = side0 & (1u << i);
            const int L = on0 ? L0 : L1;
            const int off = on0 ? 0 : L0;
            const double g = __dmul_ru(on0 ? fS : fC, small_to_double((uint32_t)L));
            const uint32_t slot = (uint32_t)__double2loint(__dadd_rz(g, 0x1p52)) + (uint32_t)off;
            const uint32_t u = cumB - slot * 0x01010101u;            // bit 7 of byte b: C_<=b > slot
            const uint32_t dm = (u >> 7) & 0x01010101u;              // one per group >= grp
            const uint32_t ssel = (uint32_t)__dp4a((int)dm, -1, 7);          // grp + 3
            const uint32_t esel = (uint32_t)__dp4a((int)dm, -1, 0x5554);     // 0x5550 + grp
            const uint32_t stB = __byte_perm(0x7F7F7F7Fu, cumB, ssel);       // 0x7F7F7F7F + C_<grp
            const uint32_t enB = __byte_perm(cumB, 0x7F7F7F7Fu + (uint32_t)(24 - i), esel);
            const uint32_t cnt = min(enB - stB, 31u);                        // in 1..24
            const uint32_t stl = stB - 0x7F7F7F7Fu - (uint32_t)off;
            const double fn = __dmul_ru(__dadd_ru(g, -small_to_double(stl)), S.invc[cnt]);
            if (on0) fS = fn; else fC = fn;
            cumB -= dm;                                              // groups >= grp lose one item
            L0 -= on0 ? 1 : 0;
            L1 -= on0 ? 0 : 1;
            sel[i >> 2] += ssel << (4 * (i & 3));                    // nibble = grp (bias -0x3333)
        }
        // 5. magnitudes, sign flags, signs
        uint32_t mag[6], F = 0;
#pragma unroll
        for (int q2 = 0; q2 < 6; q2++) {
            mag[q2] = __byte_perm(R.vals, (uint32_t)R.val4, sel[q2]);
            F |= bytes_to_nibble(__byte_perm(R.gflag, (uint32_t)R.gflag4, sel[q2])) << (4 * q2);
        }
        apply_signs(odd, word, s, F, (uint32_t)(R.flags >> 1), mag, ok, S.pdep_off, S.pdep, v);
        return ok;
    }
};

}  // namespace llvq
