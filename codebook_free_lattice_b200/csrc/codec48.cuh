// codec48.cuh -- decoder for the 48-bit index budget (2 bits per weight: shells 2..13,
// 383 classes), one thread per 24-weight block.
//
// Method: "Leech Lattice Vector Quantization for Efficient LLM Compression", papernotes.org
// notes, 方法详解 / 关键设计 2 (shell and class by cumulative offsets; r = I_class mod A,
// I' = floor(I_class / A), s = I' mod 2^B, I'' = floor(I' / 2^B)).
//
//   1. class: a guide table on the top index bits gives the candidate classes, almost always one
//      or two, decided by comparing with the class starts;
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
//      is exact.  The loop stays on the FMA, ALU and fp64 pipes.  Most even classes skip the
//      loop: p_S and p_C index precomputed arrangement tables of the two coordinate sets;
//   5. magnitudes and sign flags by byte permutation of the class's group tables, then signs.
//
// The per-class constants are stored one array per field, so that a warp reading one field for
// 32 different classes spreads over the shared-memory banks.
#pragma once
#include "device_common.cuh"

namespace llvq {

constexpr int kClasses48 = 384;
constexpr int kGuideBits48 = 12;                  // 4096 buckets over [0, 2^48)
constexpr int kGuideShift48 = 48 - kGuideBits48;

// c_info: A (bits 0..12) | B (13..17) | odd coset (18) | parity target sum|x|/4 odd (19) |
//         table path (20) | shell m (21..24) | magnitude of group 4 (25..28) | its sign flag (29)
constexpr uint32_t kInfoOdd = 1u << 18;
constexpr uint32_t kInfoParity = 1u << 19;
constexpr uint32_t kInfoTable = 1u << 20;
__host__ __device__ constexpr uint32_t info_A(uint32_t i) { return i & 0x1FFFu; }
__host__ __device__ constexpr uint32_t info_B(uint32_t i) { return (i >> 13) & 0x1Fu; }
__host__ __device__ constexpr int info_m(uint32_t i) { return (int)((i >> 21) & 0xFu); }
__host__ __device__ constexpr uint32_t info_val4(uint32_t i) { return (i >> 25) & 0xFu; }
__host__ __device__ constexpr uint32_t info_flag4(uint32_t i) { return (i >> 29) & 1u; }
// c_info2: first by-weight Golay slot of weight k (bits 0..11) | places on S: k or 24 (12..16) |
//          table path: arrangements on S, P_S (17..27)
// c_offs:  table path: first entry of the complement's table (bits 0..18) | of S's table (19..31)

constexpr int kTabS48 = 8192;                     // S-side arrangement entries (7964 used)

// Shared-memory image of the 48-bit decode tables (one copy per CTA, 70 KB).  16-byte aligned
// size: it is copied in 16-byte units, and tables placed after it are read in 16-byte units.
struct alignas(16) Smem48 {
    uint32_t golay_mask[4096];
    uint32_t golay_weight[4096];
    double invc[32];                              // 1/c rounded up, c = 1..24
    unsigned long long starts[400];               // class starts, [nclasses] = N_M
    double c_invA[kClasses48];                    // 1/A rounded up
    double c_invP[kClasses48];                    // 1/P rounded up
    double c_PC[kClasses48];                      // arrangements off S (even; exact), 1 for odd
    uint32_t c_info[kClasses48];
    uint32_t c_info2[kClasses48];
    uint32_t c_offs[kClasses48];
    uint32_t c_cum[kClasses48];                   // bytes: cumulative counts C_<=g, g = 0..3 (sat. 24)
    uint32_t c_vals[kClasses48];                  // bytes: magnitudes of groups 0..3
    uint32_t c_gflag[kClasses48];                 // bytes: per-group sign flag (odd: |x| = 1 mod 4;
                                                  //        even: |x| != 0)
    unsigned long long c_vt[kClasses48];          // odd: signed int8 value of groups 0..4 on T
    unsigned long long c_vn[kClasses48];          // odd: signed int8 value of groups 0..4 off T
    uint16_t guide[(1 << kGuideBits48) + 1];
    uint16_t pdep_off[256];
    uint8_t pdep[kPdepEntries];
    float invnorm[16];                            // 1 / (4 sqrt(m))
};

// Tables of the even-coset table path.  An arrangement entry lists the value codes of one
// coordinate set in ascending position, two bits each (code = (|x| - 2)/4 on S, |x|/4 off S),
// in lexicographic order per multiset of codes.  merge[mq << 8 | bits] places the next symbols of
// the two sets on the four coordinates of one nibble whose S positions are mq: bits holds the
// popcount(mq) S symbols, then the C symbols; the entry is the four magnitude bytes with the
// nibble's nonzero mask in bits 28..31.
struct alignas(16) SmemEven48 {
    uint32_t tabS[kTabS48];
    uint32_t merge[4096];
};
static_assert(sizeof(Smem48) % 16 == 0 && sizeof(SmemEven48) % 16 == 0, "16-byte table images");

// Steps 1-2 of the decode: the class of one packed word and its digits r, s and p = I''.
struct Cls48 {
    unsigned long long p;      // arrangement rank I''
    uint32_t r, s;             // Golay refinement, sign bits
    uint32_t info;             // c_info of the class
    int cls;                   // class index
    bool ok;                   // index < N_M (otherwise the digits describe index 0)
};

template <class Img>
__device__ __forceinline__ Cls48 classify48(unsigned long long w, const Img &S, unsigned long long npoints) {
    Cls48 c;
    unsigned long long idx = w & 0xFFFFFFFFFFFFull;
    c.ok = idx < npoints;
    if (!c.ok) idx = 0;
    // 1. class: the guide bucket of the top index bits holds classes lo..hi; almost always
    //    hi <= lo + 1, decided by one comparison; wider buckets take a binary search
    const uint32_t b = (uint32_t)(idx >> kGuideShift48);
    int lo = S.guide[b];
    const int hi = S.guide[b + 1];
    if (hi > lo + 1) {
        int h = hi;
        while (lo < h) {
            const int mid = (lo + h + 1) >> 1;
            if (S.starts[mid] <= idx) lo = mid; else h = mid - 1;
        }
    } else {
        lo += (hi > lo && S.starts[hi] <= idx) ? 1 : 0;
    }
    c.cls = lo;
    c.info = S.c_info[lo];
    const uint32_t A = info_A(c.info), B = info_B(c.info);
    // 2. I_class = r + A (s + 2^B I'').  I_class < 2^48 is exact as the double 2^52 + I_class
    //    minus 2^52; q = floor(I_class / A) comes from the product with 1/A rounded up (q or
    //    q + 1) and one correction, its 2^52-biased double giving q's bits directly.
    const unsigned long long Ic = idx - S.starts[lo];
    const double Icd = __hiloint2double(0x43300000 | (int)(Ic >> 32), (int)(uint32_t)Ic) - 0x1p52;
    const double t = __dadd_rz(__dmul_ru(Icd, S.c_invA[lo]), 0x1p52);
    uint32_t q_lo = (uint32_t)__double2loint(t);
    uint32_t q_hi = (uint32_t)__double2hiint(t) & 0xFFFFFu;
    int rem = (int)((uint32_t)Ic - q_lo * A);
    if (rem < 0) {
        rem += (int)A;
        q_hi -= q_lo == 0u ? 1u : 0u;
        q_lo -= 1u;
    }
    c.r = (uint32_t)rem;
    c.s = q_lo & ((1u << B) - 1u);
    c.p = ((unsigned long long)q_hi << 32 | q_lo) >> B;
    return c;
}

// Step 5 after the arrangement: magnitudes and sign flags from the class's group tables by the
// recorded group nibbles, then the signs.
template <class Img>
__device__ __forceinline__ void finish48(const Img &S, int cls, uint32_t info, bool odd, uint32_t word,
                                         uint32_t s, bool ok, const uint32_t sel[6], uint32_t v[6]) {
    const uint32_t vals = S.c_vals[cls], gflag = S.c_gflag[cls];
    const uint32_t val4 = info_val4(info), flag4 = info_flag4(info);
    uint32_t mag[6], F = 0;
#pragma unroll
    for (int q2 = 0; q2 < 6; q2++) {
        mag[q2] = __byte_perm(vals, val4, sel[q2]);
        F |= bytes_to_nibble(__byte_perm(gflag, flag4, sel[q2])) << (4 * q2);
    }
    apply_signs(odd, word, s, F, (info & kInfoParity) ? 1u : 0u, mag, ok, S.pdep_off, S.pdep, v);
}

// Steps 4-5 for any class, given its codeword (step 3): the arrangement of both coordinate sets,
// signs.
template <class Img>
__device__ __forceinline__ void arrange48_word(const Img &S, int cls, uint32_t info, uint32_t word,
                                               unsigned long long p, uint32_t s, bool ok, uint32_t v[6]) {
    const uint32_t info2 = S.c_info2[cls];
    const int nS = (int)((info2 >> 12) & 0x1Fu);
    const bool odd = info & kInfoOdd;
    const uint32_t side0 = odd ? 0xFFFFFFu : word;
    // 4. arrangement.  Byte b of cumB is 0x7F + C_<=b (remaining items of groups 0..b),
    //    biased one below the guard bit so the byte-wise subtraction of the slot never borrows.
    double fC = __dmul_ru((double)p, S.c_invP[cls]);            // (p_C + p_S/P_S) / P_C
    const double g0 = __dmul_ru(fC, S.c_PC[cls]);                 // p_C + p_S/P_S
    double fS = __dadd_ru(g0, 0x1p52 - __dadd_rz(g0, 0x1p52));   // p_S / P_S
    uint32_t cumB = S.c_cum[cls] + 0x7F7F7F7Fu;
    int L0 = nS, L1 = 24 - nS;
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
    finish48(S, cls, info, odd, word, s, ok, sel, v);
}

// Steps 3-5 for any class: codeword from the shared-memory Golay tables, then the arrangement.
__device__ __forceinline__ void arrange48(const Smem48 &S, int cls, uint32_t info, unsigned long long p,
                                          uint32_t r, uint32_t s, bool ok, uint32_t v[6]) {
    const uint32_t info2 = S.c_info2[cls];
    const bool odd = info & kInfoOdd;
    const uint32_t word = odd ? S.golay_mask[r & 4095u] : S.golay_weight[min((info2 & 0xFFFu) + r, 4095u)];
    arrange48_word(S, cls, info, word, p, s, ok, v);
}

// One coordinate of the odd-class loop: at coordinate i the set has 24 - i places left and the
// slot needs no offset.
__device__ __forceinline__ void odd_step48(int i, double &f, uint32_t &cumB, uint32_t sel[6], const double *invc) {
    const double g = __dmul_ru(f, (double)(24 - i));
    const uint32_t slot = (uint32_t)__double2loint(__dadd_rz(g, 0x1p52));
    const uint32_t u = cumB - slot * 0x01010101u;
    const uint32_t dm = (u >> 7) & 0x01010101u;
    const uint32_t ssel = (uint32_t)__dp4a((int)dm, -1, 7);
    const uint32_t esel = (uint32_t)__dp4a((int)dm, -1, 0x5554);
    const uint32_t stB = __byte_perm(0x7F7F7F7Fu, cumB, ssel);
    const uint32_t enB = __byte_perm(cumB, 0x7F7F7F7Fu + (uint32_t)(24 - i), esel);
    const uint32_t cnt = min(enB - stB, 31u);
    const uint32_t stl = stB - 0x7F7F7F7Fu;
    f = __dmul_ru(__dadd_ru(g, -small_to_double(stl)), invc[cnt]);
    cumB -= dm;
    sel[i >> 2] += ssel << (4 * (i & 3));
}

// The last coordinate: one place left, so the slot is 0 and the group is the one item left.
__device__ __forceinline__ void odd_last_step48(uint32_t cumB, uint32_t sel[6]) {
    const uint32_t dm = (cumB >> 7) & 0x01010101u;
    sel[5] += (uint32_t)__dp4a((int)dm, -1, 7) << 12;
}

// Steps 3-5 for an odd class only: one coordinate set, so the places left at coordinate i are
// 24 - i and the slot needs no offset.  x_i = a_i exactly when (i in T) equals (a_i = 1 mod 4),
// so each group has one signed value on T and one off T: a byte permutation of each table by the
// group nibbles, then a byte select by T.
__device__ __forceinline__ void arrange_odd48(const Smem48 &S, int cls, uint32_t info, unsigned long long p,
                                              uint32_t r, uint32_t v[6]) {
    const uint32_t T = S.golay_mask[r & 4095u];
    double f = __dmul_ru((double)p, S.c_invP[cls]);
    uint32_t cumB = S.c_cum[cls] + 0x7F7F7F7Fu;
    uint32_t sel[6] = {0u - 0x3333u, 0u - 0x3333u, 0u - 0x3333u,
                       0u - 0x3333u, 0u - 0x3333u, 0u - 0x3333u};
#pragma unroll
    for (int i = 0; i < 23; i++) odd_step48(i, f, cumB, sel, S.invc);
    odd_last_step48(cumB, sel);
    const unsigned long long vt = S.c_vt[cls], vn = S.c_vn[cls];
#pragma unroll
    for (int q = 0; q < 6; q++) {
        const uint32_t pt = __byte_perm((uint32_t)vt, (uint32_t)(vt >> 32), sel[q]);
        const uint32_t pn = __byte_perm((uint32_t)vn, (uint32_t)(vn >> 32), sel[q]);
        const uint32_t tb = nibble_to_bytes((T >> (4 * q)) & 0xFu) * 0xFFu;     // 0xFF on T
        v[q] = (pt & tb) | (pn & ~tb);
    }
}

// Step 4 for an even class on the table path: p_C = floor(f_C P_C) and p_S from the scaled
// fraction as in the loop; they index the arrangement tables of the complement and of S.
struct Even48Idx {
    uint32_t pC, pS;
};
template <class Img>
__device__ __forceinline__ Even48Idx even48_indices(const Img &S, int cls, unsigned long long p) {
    Even48Idx x;
    const double fC = __dmul_ru(small_to_double((uint32_t)p), S.c_invP[cls]);   // (p_C + p_S/P_S) / P_C
    const double g0 = __dmul_ru(fC, S.c_PC[cls]);                               // p_C + p_S/P_S
    const double t0 = __dadd_rz(g0, 0x1p52);                                    // 2^52 + p_C
    x.pC = (uint32_t)__double2loint(t0);
    const double fS = __dadd_ru(g0, 0x1p52 - t0);                               // p_S / P_S
    const double h = __dmul_ru(fS, small_to_double(S.c_info2[cls] >> 17));
    x.pS = (uint32_t)__double2loint(__dadd_rz(h, 0x1p52));
    return x;
}

// Step 5 for an even class on the table path, given its codeword and the two sets' code sequences:
// the sequences merged nibble by nibble along the codeword, then the signs.
template <class Img>
__device__ __forceinline__ void even48_merge_word(const Img &S, const uint32_t *merge, uint32_t info, uint32_t word,
                                                  uint32_t s, uint32_t sS, uint32_t cS, uint32_t v[6]) {
    uint32_t mag[6], F = 0, Sw = word;
#pragma unroll
    for (int q = 0; q < 6; q++) {
        const uint32_t mq = Sw & 0xFu;
        Sw >>= 4;
        const uint32_t n2 = 2u * (uint32_t)__popc(mq);
        const uint32_t bits = ((sS & ((1u << n2) - 1u)) | (cS << n2)) & 0xFFu;
        const uint32_t e = merge[(mq << 8) | bits];
        mag[q] = e & 0x0F0F0F0Fu;
        F |= (e >> 28) << (4 * q);
        sS >>= n2;
        cS >>= 8u - n2;
    }
    apply_signs(false, word, s, F, (info & kInfoParity) ? 1u : 0u, mag, true, S.pdep_off, S.pdep, v);
}

// Steps 3 and 5 for an even class on the table path: the codeword S from the shared-memory table,
// then the merge.
__device__ __forceinline__ void even48_merge(const Smem48 &S, const SmemEven48 &E, uint32_t info, uint32_t info2,
                                             uint32_t r, uint32_t s, uint32_t sS, uint32_t cS, uint32_t v[6]) {
    const uint32_t word = S.golay_weight[min((info2 & 0xFFFu) + r, 4095u)];
    even48_merge_word(S, E.merge, info, word, s, sS, cS, v);
}

// Steps 3-5 for an even class on the table path.
__device__ __forceinline__ void arrange_even48_table(const Smem48 &S, const SmemEven48 &E,
                                                     const uint32_t *__restrict__ tabC, int cls, uint32_t info,
                                                     unsigned long long p, uint32_t r, uint32_t s, uint32_t v[6]) {
    const Even48Idx x = even48_indices(S, cls, p);
    const uint32_t offs = S.c_offs[cls];
    const uint32_t cS = __ldg(tabC + (offs & 0x7FFFFu) + x.pC);
    even48_merge(S, E, info, S.c_info2[cls], r, s, E.tabS[(offs >> 19) + x.pS], cS, v);
}

struct Dec48 {
    using Word = unsigned long long;
    using Smem = Smem48;
    struct Args {
        const Smem48 *image;
        unsigned long long npoints;
    };
    static constexpr int kWordBytes = 8;
    static constexpr int kCtasPerSm = 3;          // 40 registers, 70 KB shared per CTA

    __device__ static Word load(const Word *p) { return __ldg(p); }
    __device__ static int gain_code(const Word &w) { return (int)((w >> 48) & 0xFFu); }
    __device__ static float invnorm(const Smem &S, int m) { return S.invnorm[m]; }

    // Decode one packed word into 24 signed int8 coordinates (v[q] byte b = coordinate 4q+b).
    // Returns false (and v = 0) for an index >= N_M.  m receives the shell.
    __device__ static bool decode(const Word &w, const Smem &S, const Args &a, uint32_t v[6], int &m) {
        const Cls48 c = classify48(w, S, a.npoints);
        m = info_m(c.info);
        arrange48(S, c.cls, c.info, c.p, c.r, c.s, c.ok, v);
        return c.ok;
    }
};

}  // namespace llvq

namespace llvq {

// ---- odd-coset decode producing fp16 weights (fused products) --------------------------------
//
// The odd class's arrangement rank is unranked by the same exact arithmetic decoding as above,
// restated for the product path so that each coordinate costs fewer instructions:
//   * the group search yields, by one byte permutation, the biased bytes (31 + C_<a, 31 + C_<=a)
//     of the chosen group a; the start and the count c follow by two byte dot products;
//   * each coordinate emits a byte-permutation selector (nibbles 2a, 2a + 1) that later picks
//     the group's fp16 value from an 8-byte table;
//   * the last 6 coordinates come from one shared-memory table: the 4^6 arrangements of every
//     multiset of 6 items over 4 groups, lexicographic per multiset (2-bit group codes), indexed by
//     the multiset (its cumulative counts) and floor(f * arrangements).
// Only classes with at most 4 magnitude groups take this path.

constexpr int kOddTail48 = 6;                                  // coordinates taken from the tail table
constexpr int kOddSteps48 = 24 - kOddTail48;                   // coordinates decoded step by step
constexpr int kOddBias48 = 31;                                 // byte bias of the cumulative counts

// Shared-memory image of the fused product kernel (k_gemv48): what classification, the odd-coset
// fp16 path, the even-coset table path and the rare generic path read per block.  An odd codeword
// is computed from r; the complement arrangement table (1.6 MB) is read from global memory.
//
// merge16[mq << 8 | bits] serves the even-coset fp16 path: for the four coordinates of one nibble
// whose codeword positions are mq, bits holds the popcount(mq) S-side codes and then the
// complement codes (2 bits each, in position order); the entry is the byte-permutation selectors
// of the coordinates' fp16 values as two pairs, (z0, i0, z1, i1) and (z2, i2, z3, i3), where i is
// |x| / 2, an index into the 8-byte table of the fp16 high bytes of 0, 2, ..., 14, and z is the
// nibble 0 or 8 (both give the zero low byte), bit 3 of z_k being the coordinate's nonzero flag.
struct alignas(16) SmemGv48 {
    unsigned long long starts[400];               // class starts, [nclasses] = N_M
    double c_invA[kClasses48];                    // 1/A rounded up
    double c_invP[kClasses48];                    // 1/P rounded up
    double c_PC[kClasses48];                      // arrangements off S (even; exact), 1 for odd
    double invc[32];                              // 1/c rounded up, c = 1..24
    uint32_t c_info[kClasses48];
    uint32_t c_info2[kClasses48];
    uint32_t c_offs[kClasses48];
    uint32_t c_cum[kClasses48];                   // bytes: cumulative counts C_<=g, g = 0..3 (sat. 24)
    uint32_t c_vals[kClasses48];                  // bytes: magnitudes of groups 0..3
    uint32_t c_gflag[kClasses48];                 // bytes: per-group sign flag
    uint32_t c_cumodd[kClasses48];                // odd, <= 4 groups: bytes 31 + C_<=g, g = 0..3
    uint32_t c_vt[kClasses48][2];                 // odd, <= 4 groups: fp16 value of groups 0..3 on T
    uint32_t c_magS[kClasses48];                  // even table path: ceil(2^32 / P_S), 0 for P_S = 1
    float invnorm[16];                            // 1 / (4 sqrt(m))
    uint32_t merge16[4096];                       // even table path (see above)
    uint32_t tabS[kTabS48];                       // even table path: S-side code sequences (see SmemEven48)
    uint32_t gweight[4096];                       // Golay codewords in (weight, mask) order
    uint2 nsign[16];                              // for a nibble of negative flags: the two coordinate-pair masks
    uint2 tailc[344];                             // [C<=0 + 7 C<=1 + 49 C<=2] of a 6-item multiset: (first entry, count)
    uint16_t tail[4096];                          // the 6-item arrangements, 2-bit group codes, first coordinate lowest
    uint16_t guide[(1 << kGuideBits48) + 8];
    uint16_t tlow[128];                           // low 12 bits of the codeword whose top 12 bits are r: [r & 63] ^ [64 + (r >> 6)]
    uint16_t pdep_off[256];
    uint8_t pdep[kPdepEntries + 15];
};
static_assert(sizeof(SmemGv48) % 16 == 0, "16-byte table image");

// The codeword T of an odd class: the codeword whose top 12 bits are r (coordinates 12..23 are an
// information set of this Golay code, and codewords in mask order ascend by their top bits).
__device__ __forceinline__ uint32_t odd_codeword48(const SmemGv48 &S, uint32_t r) {
    return r << 12 | (uint32_t)(S.tlow[r & 63u] ^ S.tlow[64u + (r >> 6)]);
}

// PTX prmt in its generic mode: a selector nibble with bit 3 set replicates the sign of the byte.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// One coordinate of the odd-class decode.  cum bytes: 31 + C_<=b of the remaining items.  One
// byte permutation of (31 << 24, cum) gives (31 + C_<a, 31 + C_<=a) of the chosen group a
// (C_<0 = 0 comes from the constant's top byte); then f <- (f L - C_<a) / c rounded upward.
// sel[i / 4] byte i % 4 receives 0x10 + 0x22 a (fp16 selector of group a).
template <int I>
__device__ __forceinline__ void odd_step_f16(double &f, uint32_t &cum, uint32_t sel[6], const double *invc) {
    constexpr double L = (double)(24 - I);
    const double g = __dmul_ru(f, L);
    const uint32_t slot = (uint32_t)__double2loint(__dadd_rz(g, 0x1p52));
    const uint32_t u = cum - slot * 0x01010101u;                 // bit 5 of byte b: C_<=b > slot
    const uint32_t dm = (u >> 5) & 0x01010101u;                  // one per group b >= a
    const uint32_t osel = (uint32_t)__dp4a((int)dm, (int)0xDEDEDEDE, 0x98);     // 0x10 + 0x22 a
    const uint32_t psel = (uint32_t)__dp4a((int)dm, (int)0xEFEFEFEF, 0x8887);   // 3 + a, 4 + a, zero, zero
    const uint32_t r = prmt(0x1F000000u, cum, psel);             // (31 + C_<a) | (31 + C_<=a) << 8
    const uint32_t c = (uint32_t)__dp4a((int)r, 0x000001FF, 0);  // C_<=a - C_<a
    const int st = __dp4a((int)r, 1, -kOddBias48);               // C_<a
    const double d = __dadd_ru(g, -(__hiloint2double(0x43300000, st) - 0x1p52));
    f = __dmul_ru(d, invc[c]);
    cum -= dm;
    sel[I >> 2] += osel << (8 * (I & 3));
}

// Steps 3-5 of an even class on the table path, as fp16 pairs v[q] (coordinates 2q, 2q + 1):
// p = p_S + P_S p_C by one multiply-high and a correction; the complement's code sequence from
// the global table cS (its entry fetched by the caller), the S side from shared memory; the two
// sequences merged nibble by nibble into fp16 selectors (merge16), with the nonzero flags F; the
// sign bits s deposited on the nonzero coordinates skipping the highest of S, whose sign makes the
// number of negatives on S match the class parity; signs applied to the fp16 pairs.
__device__ __forceinline__ uint32_t even48_pC(const SmemGv48 &S, int cls, uint32_t p, uint32_t &pS) {
    const uint32_t PS = S.c_info2[cls] >> 17, m = S.c_magS[cls];
    uint32_t q = m ? __umulhi(p, m) : p;                  // q or q + 1
    int rem = (int)(p - q * PS);
    if (rem < 0) {
        rem += (int)PS;
        q -= 1u;
    }
    pS = (uint32_t)rem;
    return q;
}
__device__ __forceinline__ void arrange_even48_f16(const SmemGv48 &S, int cls, uint32_t info, uint32_t pS,
                                                   uint32_t r, uint32_t s, uint32_t cS, uint32_t v[12]) {
    const uint32_t offs = S.c_offs[cls];
    const uint32_t info2 = S.c_info2[cls];
    uint32_t sS = S.tabS[(offs >> 19) + pS];
    const uint32_t word = S.gweight[min((info2 & 0xFFFu) + r, 4095u)];
    constexpr uint32_t kVlo = 0x46444000u, kVhi = 0x4B4A4948u;   // fp16 high bytes of 0, 2, ..., 14
    uint32_t Sw = word, F = 0;
#pragma unroll
    for (int q = 0; q < 6; q++) {
        const uint32_t mq = Sw & 0xFu;
        Sw >>= 4;
        const uint32_t n2 = 2u * (uint32_t)__popc(mq);
        const uint32_t bits = ((sS & ((1u << n2) - 1u)) | (cS << n2)) & 0xFFu;
        const uint32_t e = S.merge16[(mq << 8) | bits];
        sS >>= n2;
        cS >>= 8u - n2;
        v[2 * q] = prmt(kVlo, kVhi, e);
        v[2 * q + 1] = prmt(kVlo, kVhi, e >> 16);
        F |= (((e & 0x08080808u) * 0x01020408u) >> 27) << (4 * q);
    }
    const uint32_t topbit = word ? (0x80000000u >> __clz(word)) : 0u;
    uint32_t neg = pdep24(s, F & ~topbit, S.pdep_off, S.pdep);
    neg |= ((__popc(neg & word) ^ ((info & kInfoParity) ? 1u : 0u)) & 1u) ? topbit : 0u;
#pragma unroll
    for (int q = 0; q < 6; q++) {
        const uint2 m = S.nsign[(neg >> (4 * q)) & 0xFu];
        v[2 * q] ^= m.x;
        v[2 * q + 1] ^= m.y;
    }
}

// Steps 3-5 of an odd class on the fp16 path: the 24 coordinates as fp16 pairs v[q] (coordinates
// 2q, 2q + 1), signs included.
__device__ __forceinline__ void odd48_setup(const SmemGv48 &S, int cls, unsigned long long p, double &f,
                                            uint32_t &cum, uint32_t sel[6]) {
    f = __dmul_ru(__hiloint2double(0x43300000 | (int)(uint32_t)(p >> 32), (int)(uint32_t)p) - 0x1p52, S.c_invP[cls]);
    cum = S.c_cumodd[cls];
#pragma unroll
    for (int q = 0; q < 6; q++) sel[q] = 0u;
}
// the last 6 coordinates from the tail table: multiset by its cumulative counts, rank
// floor(f * count); the 2-bit group codes spread to nibbles, then to fp16 selectors (0x10 + 0x22 a
// by a byte permutation); then the values (the group's fp16 value on T, negated off T)
__device__ __forceinline__ void odd48_finish(const SmemGv48 &S, int cls, uint32_t r, double f, uint32_t cum,
                                             uint32_t sel[6], uint32_t v[12]) {
    const uint32_t cid = (uint32_t)__dp4a((int)cum, 0x00310701, -kOddBias48 * 57);
    const uint2 tc = S.tailc[cid];
    const double cnt = __hiloint2double(0x43300000, (int)tc.y) - 0x1p52;
    const uint32_t rank = (uint32_t)__double2loint(__dadd_rz(__dmul_ru(f, cnt), 0x1p52));
    uint32_t x = S.tail[tc.x + rank];                       // codes of coordinates 18..23
    x = (x | x << 8) & 0x00FF00FFu;
    x = (x | x << 4) & 0x0F0F0F0Fu;
    x = (x | x << 2) & 0x33333333u;                         // nibble k: code of coordinate 18 + k
    sel[4] |= prmt(0x76543210u, 0u, x) << 16;               // coordinates 18, 19 into bytes 2, 3
    sel[5] = prmt(0x76543210u, 0u, x >> 8);                 // coordinates 20..23
    const uint32_t offT = ~odd_codeword48(S, r);
    const uint32_t vt0 = S.c_vt[cls][0], vt1 = S.c_vt[cls][1];
#pragma unroll
    for (int b = 0; b < 3; b++) {
        const uint2 m0 = S.nsign[(offT >> (8 * b)) & 0xFu], m1 = S.nsign[(offT >> (8 * b + 4)) & 0xFu];
        const uint32_t s0 = sel[2 * b], s1 = sel[2 * b + 1];
        v[4 * b + 0] = prmt(vt0, vt1, s0) ^ m0.x;
        v[4 * b + 1] = prmt(vt0, vt1, s0 >> 16) ^ m0.y;
        v[4 * b + 2] = prmt(vt0, vt1, s1) ^ m1.x;
        v[4 * b + 3] = prmt(vt0, vt1, s1 >> 16) ^ m1.y;
    }
}
#define LLVQ_ODD_STEPS(X)                                                                         \
    X(0) X(1) X(2) X(3) X(4) X(5) X(6) X(7) X(8) X(9) X(10) X(11) X(12) X(13) X(14) X(15) X(16) X(17)
__device__ __forceinline__ void arrange_odd48_f16(const SmemGv48 &S, int cls, unsigned long long p, uint32_t r,
                                                  uint32_t v[12]) {
    double f;
    uint32_t cum, sel[6];
    odd48_setup(S, cls, p, f, cum, sel);
#define LLVQ_STEP1(I) odd_step_f16<I>(f, cum, sel, S.invc);
    LLVQ_ODD_STEPS(LLVQ_STEP1)
#undef LLVQ_STEP1
    odd48_finish(S, cls, r, f, cum, sel, v);
}
}  // namespace llvq
