// llvq.cu -- LLVQ decode and fused decode-and-multiply kernels for B200 (sm_100a), with the
// C ABI declared in include/llvq.h.
//
// Method ("Leech Lattice Vector Quantization for Efficient LLM Compression"):
//   papernotes.org notes, 方法详解 / 关键设计 2 -- the hierarchical bijection: shell by
//     cumulative offsets, class by class offsets, then r = I_class mod A, I' = floor(I_class/A),
//     s = I' mod 2^B, I'' = floor(I'/2^B) (Golay refinement, sign pattern, lexicographic rank);
//   关键设计 4 -- fused dequantize-and-multiply: decode in registers/shared memory, dot with the
//     activations, never write dequantized weights to global memory;
//   gist.science summary, Methodik 4 -- a fully parallel decode by modular arithmetic.
//
// Decode of one 48-bit index (one thread per block of 24 weights):
//   1. class search: a guide table on the top index bits narrows a binary search over the
//      class start offsets (shared memory);
//   2. r, s, I'' by one fp64 division by A with an exact integer correction;
//   3. codeword from the shared-memory Golay tables;
//   4. the lexicographic rank I'' is unranked coordinate by coordinate, in coordinate order,
//      as exact arithmetic decoding: f = I''/P in fp64 rounded upward; at a coordinate of side
//      sigma with L remaining places, the slot floor(f * L) selects the magnitude group among
//      the side's remaining items (byte-SIMD search of the cumulative counts), and
//      f <- (f * L - start(group)) / count(group).  Directed rounding keeps f above the exact
//      value with an error far below 1/(remaining arrangements) (P < 2^33 at 48 bits), so
//      every slot is exact;
//   5. signs in bulk (odd coset from the codeword T, even coset by depositing s on the
//      nonzero coordinates), then the dot product / store.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/llvq.h"
#include "tables.h"

namespace llvq {

// --------------------------------------------------------------------------------------
// device records
// --------------------------------------------------------------------------------------
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
};
static_assert(sizeof(Rec48) == 48, "Rec48 layout");

constexpr int kGuideBits48 = 11;                  // 2048 buckets over [0, 2^48)
constexpr int kGuideShift48 = 48 - kGuideBits48;
constexpr int kPdepEntries = 6561;                // sum over 8-bit masks of 2^popcount

// Shared-memory image of the 48-bit decode tables (one copy per CTA).
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

struct Dev48 {                                    // global-memory master copy
    Smem48 *image;                                // bytes to copy into shared memory
    int nclasses;
    unsigned long long npoints;
};

// --------------------------------------------------------------------------------------
// device helpers
// --------------------------------------------------------------------------------------
__device__ __forceinline__ void load_smem_image(void *dst, const void *src, size_t bytes) {
    const int4 *s = reinterpret_cast<const int4 *>(src);
    int4 *d = reinterpret_cast<int4 *>(dst);
    size_t n = bytes / 16;
    for (size_t i = threadIdx.x; i < n; i += blockDim.x) d[i] = __ldg(s + i);
}

// bit k of the nibble -> byte k (0x01)
__device__ __forceinline__ uint32_t nibble_to_bytes(uint32_t nib) {
    return (nib * 0x00204081u) & 0x01010101u;
}
// byte k's bit 0 -> bit k of a nibble
__device__ __forceinline__ uint32_t bytes_to_nibble(uint32_t b) {
    return ((b & 0x01010101u) * 0x01020408u) >> 24 & 0xFu;
}

// exact double of a small non-negative integer (n < 2^31) without a conversion instruction
__device__ __forceinline__ double small_to_double(uint32_t n) {
    return __hiloint2double(0x43300000, (int)n) - 0x1p52;
}

// deposit the low bits of src on the set bits of mask (24-bit), lowest first
__device__ __forceinline__ uint32_t pdep24(uint32_t src, uint32_t mask, const Smem48 &S) {
    uint32_t out = 0;
#pragma unroll
    for (int j = 0; j < 3; j++) {
        uint32_t mb = (mask >> (8 * j)) & 0xFFu;
        uint32_t n = __popc(mb);
        uint32_t bits = src & ((1u << n) - 1u);
        out |= (uint32_t)S.pdep[S.pdep_off[mb] + bits] << (8 * j);
        src >>= n;
    }
    return out;
}

// Decode one 48-bit index into 24 signed int8 coordinates packed in v[6] (coordinate 4q+b in
// byte b of v[q]).  Returns false (and v = 0) if idx >= N_M.  m receives the shell.
__device__ __forceinline__ bool decode48(unsigned long long idx, const Smem48 &S,
                                         unsigned long long npoints, int nclasses, uint32_t v[6],
                                         int &m) {
    const bool ok = idx < npoints;
    if (!ok) idx = 0;
    // 1. class: guide bucket, then binary search of the starts
    int lo = S.guide[idx >> kGuideShift48];
    int hi = S.guide[(idx >> kGuideShift48) + 1];
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (S.starts[mid] <= idx) lo = mid; else hi = mid - 1;
    }
    const Rec48 R = S.recs[lo];
    m = R.m;
    // 2. I_class = r + A (s + 2^B I'')
    unsigned long long Ic = idx - R.start;
    unsigned long long q = (unsigned long long)((double)Ic * R.invA);
    long long rem = (long long)(Ic - q * R.A);
    if (rem < 0) { q -= 1; rem += R.A; }
    else if (rem >= (long long)R.A) { q += 1; rem -= R.A; }
    const uint32_t r = (uint32_t)rem;
    const uint32_t s = (uint32_t)(q & ((1ull << R.B) - 1ull));
    const unsigned long long p = q >> R.B;
    // 3. codeword: odd -> T (x_i = 1 mod 4 on T); even -> S (|x_i| = 2 mod 4 on S)
    const bool odd = R.flags & 1u;
    const uint32_t word = odd ? S.golay_mask[r & 4095u] : S.golay_weight[min(R.wbase + r, 4095u)];
    const uint32_t side0 = odd ? 0xFFFFFFu : word;
    // 4. arrangement, coordinate by coordinate.  Byte b of cumB is 0x7F + C_<=b (remaining
    //    items of groups 0..b, biased one below the guard bit so the byte-wise subtraction of
    //    the slot is borrow-free).  The loop keeps to the FMA, ALU and fp64 pipes: floor() by
    //    the 2^52 magic add, int -> double by building 2^52 + n, the group count by a byte dot
    //    product.
    double f = __dmul_ru((double)p, R.invP);
    uint32_t cumB = R.cum + 0x7F7F7F7Fu;
    int L0 = R.nS, L1 = 24 - R.nS;
    uint32_t sel[6] = {0u - 0x3333u, 0u - 0x3333u, 0u - 0x3333u, 0u - 0x3333u, 0u - 0x3333u, 0u - 0x3333u};
#pragma unroll
    for (int i = 0; i < 24; i++) {
        const bool on0 = side0 & (1u << i);
        const int L = on0 ? L0 : L1;
        const int off = on0 ? 0 : L0;
        const double g = __dmul_ru(f, small_to_double((uint32_t)L));
        const uint32_t slot = (uint32_t)__double2loint(__dadd_rz(g, 0x1p52)) + (uint32_t)off;
        const uint32_t u = cumB - slot * 0x01010101u;            // bit 7 of byte b: C_<=b > slot
        const uint32_t dm = (u >> 7) & 0x01010101u;              // one per group >= grp
        const uint32_t ssel = (uint32_t)__dp4a((int)dm, -1, 7);          // grp + 3
        const uint32_t esel = (uint32_t)__dp4a((int)dm, -1, 0x5554);     // 0x5550 + grp
        const uint32_t stB = __byte_perm(0x7F7F7F7Fu, cumB, ssel);       // 0x7F7F7F7F + C_<grp
        const uint32_t enB = __byte_perm(cumB, 0x7F7F7F7Fu + (uint32_t)(24 - i), esel);  // + C_<=grp
        const uint32_t cnt = min(enB - stB, 31u);                        // in 1..24
        const uint32_t stl = stB - 0x7F7F7F7Fu - (uint32_t)off;
        f = __dmul_ru(__dadd_ru(g, -small_to_double(stl)), S.invc[cnt]);
        cumB -= dm;                                              // groups >= grp lose one item
        L0 -= on0 ? 1 : 0;
        L1 -= on0 ? 0 : 1;
        sel[i >> 2] += ssel << (4 * (i & 3));                    // nibble = grp (bias -0x3333)
    }
    // 5. magnitudes and per-coordinate sign flags by byte permutation of the group tables
    uint32_t mag[6], F = 0;
#pragma unroll
    for (int qq = 0; qq < 6; qq++) {
        mag[qq] = __byte_perm(R.vals, (uint32_t)R.val4, sel[qq]);
        F |= bytes_to_nibble(__byte_perm(R.gflag, (uint32_t)R.gflag4, sel[qq])) << (4 * qq);
    }
    // 6. signs.  odd: x_i = 1 (mod 4) exactly on T, so |x_i| = 1 (mod 4) is negative off T
    //    and |x_i| = 3 (mod 4) negative on T.  even: bit j of s negates the j-th nonzero
    //    coordinate (ascending), skipping the highest coordinate of S, whose sign makes the
    //    number of negatives on S = sum|x|/4 (mod 2).
    uint32_t neg;
    if (odd) {
        neg = word ^ F;
    } else {
        const uint32_t topbit = word ? (0x80000000u >> __clz(word)) : 0u;
        neg = pdep24(s, F & ~topbit, S);
        neg |= ((__popc(neg & word) ^ (R.flags >> 1)) & 1u) ? topbit : 0u;
    }
#pragma unroll
    for (int qq = 0; qq < 6; qq++) {
        const uint32_t nb = nibble_to_bytes((neg >> (4 * qq)) & 0xFu);
        v[qq] = ok ? (mag[qq] ^ (nb * 0xFFu)) + nb : 0u;
    }
    return ok;
}

// --------------------------------------------------------------------------------------
// kernels
// --------------------------------------------------------------------------------------
__global__ void __launch_bounds__(512, 3) k_decode48(const Smem48 *__restrict__ image, int nclasses,
                                                  unsigned long long npoints,
                                                  const unsigned long long *__restrict__ words,
                                                  long long n, int8_t *__restrict__ out,
                                                  unsigned *__restrict__ flags) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem48 &S = *reinterpret_cast<Smem48 *>(smem_raw);
    load_smem_image(&S, image, sizeof(Smem48));
    __syncthreads();
    bool bad = false;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n;
         t += (long long)gridDim.x * blockDim.x) {
        const unsigned long long w = __ldg(words + t) & 0xFFFFFFFFFFFFull;
        uint32_t v[6];
        int m;
        bad |= !decode48(w, S, npoints, nclasses, v, m);
        uint2 *o = reinterpret_cast<uint2 *>(out + t * 24);
        o[0] = make_uint2(v[0], v[1]);
        o[1] = make_uint2(v[2], v[3]);
        o[2] = make_uint2(v[4], v[5]);
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicOr(flags, LLVQ_FLAG_INDEX_RANGE);
}

// Fused decode and multiply, batch BATCH (1..16).  Each CTA owns a contiguous range of rows;
// its threads walk the range's blocks in row-major order (each warp reads 32 consecutive
// packed words), decode each block once and form scale * <v, x_b> for every batch row.
// Contributions go to shared-memory accumulators acc[b][row][lane] by atomic add (the lanes of a
// warp hit distinct words, so only warps of the same CTA can meet on a word); at the end one
// warp per (b, row) sums the 32 lane slots and writes the output.
template <int BATCH>
constexpr int gemm_ctas_per_sm() { return BATCH == 1 ? 3 : 2; }

template <int BATCH>
__global__ void __launch_bounds__(512, gemm_ctas_per_sm<BATCH>()) k_gemm48(
    const Smem48 *__restrict__ image, int nclasses, unsigned long long npoints,
    const unsigned long long *__restrict__ words, long long pitch, int rows, int nb, uint32_t nb_recip,
    int gain_mode, const __half_raw *__restrict__ gains, const __half_raw *__restrict__ X,
    float *__restrict__ Y, int rows_per_cta, unsigned *__restrict__ flags) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem48 &S = *reinterpret_cast<Smem48 *>(smem_raw);
    float *acc = reinterpret_cast<float *>(smem_raw + sizeof(Smem48));   // [BATCH][rows_per_cta][32]
    load_smem_image(&S, image, sizeof(Smem48));
    for (int i = threadIdx.x; i < BATCH * rows_per_cta * 32; i += blockDim.x) acc[i] = 0.f;
    __syncthreads();
    const int row0 = blockIdx.x * rows_per_cta;
    const int nrows = min(rows_per_cta, rows - row0);
    const long long K = (long long)nb * 24;
    const int lane = threadIdx.x & 31;
    bool bad = false;
    if (nrows > 0) {
        const int total = nrows * nb;
        for (int t = threadIdx.x; t < total; t += blockDim.x) {
            // row of block t: t / nb by a multiply-high with ceil(2^32 / nb) (exact for t < 2^32 / nb)
            const int rl = nb == 1 ? t : (int)__umulhi((uint32_t)t, nb_recip);
            const int j = t - rl * nb;
            const int r = row0 + rl;
            const unsigned long long w = __ldg(words + (long long)r * pitch + j);
            uint32_t v[6];
            int m;
            bad |= !decode48(w & 0xFFFFFFFFFFFFull, S, npoints, nclasses, v, m);
            float scale;
            if (gain_mode == LLVQ_GAIN_FP16_DIRECT) {
                scale = __half2float(__ldg(reinterpret_cast<const __half *>(gains) + (long long)r * nb + j));
            } else {
                const int code = (int)((w >> 48) & 0xFFu);
                scale = __half2float(__ldg(reinterpret_cast<const __half *>(gains) + (long long)r * 256 + code)) *
                        S.invnorm[m];
            }
            float wv[24];
#pragma unroll
            for (int qq = 0; qq < 6; qq++)
#pragma unroll
                for (int e = 0; e < 4; e++) wv[4 * qq + e] = (float)(int8_t)(v[qq] >> (8 * e));
#pragma unroll
            for (int bb = 0; bb < BATCH; bb++) {
                const uint4 *xp = reinterpret_cast<const uint4 *>(X + bb * K + (long long)j * 24);
                float dot = 0.f;
#pragma unroll
                for (int c = 0; c < 3; c++) {
                    const uint4 raw = __ldg(xp + c);
                    const uint32_t h[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const float2 xf = __half22float2(*reinterpret_cast<const __half2 *>(&h[e]));
                        dot = fmaf(wv[8 * c + 2 * e], xf.x, dot);
                        dot = fmaf(wv[8 * c + 2 * e + 1], xf.y, dot);
                    }
                }
                atomicAdd(&acc[(bb * rows_per_cta + rl) * 32 + lane], scale * dot);   // lanes never collide
            }
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    for (int i = warp; i < BATCH * nrows; i += blockDim.x >> 5) {
        const int bb = i / nrows, rl = i - bb * nrows;
        float sum = acc[(bb * rows_per_cta + rl) * 32 + lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        if (lane == 0) Y[(long long)bb * rows + row0 + rl] = sum;
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicOr(flags, LLVQ_FLAG_INDEX_RANGE);
}

}  // namespace llvq

// ==========================================================================================
// host side
// ==========================================================================================
using namespace llvq;

struct llvq_codec {
    int index_bits = 0;
    int device = -1;
    int M = 0;
    u128 npoints = 0;
    int64_t nclasses = 0;
    int num_sms = 0;
    Smem48 *d_image48 = nullptr;
    unsigned *d_flags = nullptr;
};

namespace {

double round_up_recip(double c) {
    // smallest double >= 1/c
    double r = 1.0 / c;
    if (r * c < 1.0) r = std::nextafter(r, INFINITY);
    // r*c is computed with rounding; check with fma for exactness
    while (std::fma(r, c, -1.0) < 0.0) r = std::nextafter(r, INFINITY);
    return r;
}

double round_up_recip_u128(u128 P) {
    // smallest double >= 1/P (P < 2^53 at 48 bits, exact as a double)
    double d = (double)P;
    double r = 1.0 / d;
    while (std::fma(r, d, -1.0) < 0.0) r = std::nextafter(r, INFINITY);
    return r;
}

void fill_pdep(Smem48 &S) {
    int off = 0;
    for (int mb = 0; mb < 256; mb++) {
        S.pdep_off[mb] = (uint16_t)off;
        int n = __builtin_popcount(mb);
        for (int bits = 0; bits < (1 << n); bits++) {
            uint32_t outb = 0;
            int src = 0;
            for (int pos = 0; pos < 8; pos++)
                if (mb >> pos & 1) { if (bits >> src & 1) outb |= 1u << pos; src++; }
            S.pdep[off + bits] = (uint8_t)outb;
        }
        off += 1 << n;
    }
}

llvq_status build_image48(const HostTables &T, Smem48 &S, std::string &err) {
    std::memset(&S, 0, sizeof S);
    if (T.classes.size() > 383 || T.M > 15) { err = "48-bit table larger than expected"; return LLVQ_ERR_UNSUPPORTED; }
    std::memcpy(S.golay_mask, T.golay_by_mask, sizeof S.golay_mask);
    std::memcpy(S.golay_weight, T.golay_by_weight, sizeof S.golay_weight);
    S.invc[0] = 0.0;
    for (int c = 1; c < 32; c++) S.invc[c] = round_up_recip((double)c);
    const int nc = (int)T.classes.size();
    for (int i = 0; i < nc; i++) {
        const HostClass &c = T.classes[i];
        Rec48 &R = S.recs[i];
        R.start = (unsigned long long)c.start;
        R.invP = round_up_recip_u128(c.P);
        R.invA = 1.0 / (double)c.A;
        R.A = c.A;
        if (c.vals.size() > 5) { err = "more than 5 magnitude groups"; return LLVQ_ERR_UNSUPPORTED; }
        uint32_t cum = 0, vals = 0;
        int acc = 0;
        for (int g = 0; g < 4; g++) {
            if (g < (int)c.cnts.size()) acc += c.cnts[g];
            cum |= (uint32_t)std::min(acc, 24) << (8 * g);
            if (g < (int)c.vals.size()) vals |= (uint32_t)c.vals[g] << (8 * g);
        }
        uint32_t gflag = 0;
        for (int g = 0; g < 4 && g < (int)c.vals.size(); g++) {
            int v = c.vals[g];
            gflag |= (uint32_t)(c.odd ? (v % 4 == 1) : (v != 0)) << (8 * g);
        }
        R.cum = cum;
        R.vals = vals;
        R.gflag = gflag;
        R.val4 = c.vals.size() > 4 ? (uint8_t)c.vals[4] : 0;
        R.gflag4 = c.vals.size() > 4 ? (uint8_t)(c.odd ? (c.vals[4] % 4 == 1) : (c.vals[4] != 0)) : 0;
        R.nS = (uint8_t)(c.odd ? 24 : c.k);
        R.B = (uint8_t)c.B;
        R.flags = (uint8_t)((c.odd ? 1 : 0) | (((c.sum_abs / 4) & 1) << 1));
        R.wbase = (uint16_t)(c.odd ? 0 : T.weight_base[c.k]);
        R.m = (uint8_t)c.m;
        S.starts[i] = (unsigned long long)c.start;
    }
    S.starts[nc] = (unsigned long long)T.n_points;
    for (int i = nc + 1; i < 400; i++) S.starts[i] = ~0ull;
    // guide: bucket b -> class holding index b << shift (last class for buckets past N_M)
    for (int b = 0; b <= (1 << kGuideBits48); b++) {
        unsigned long long first = (unsigned long long)b << kGuideShift48;
        int lo = 0;
        while (lo + 1 < nc && S.starts[lo + 1] <= first) lo++;
        S.guide[b] = (uint16_t)lo;
    }
    fill_pdep(S);
    for (int m = 0; m < 16; m++) S.invnorm[m] = m > 0 ? (float)(1.0 / (4.0 * std::sqrt((double)m))) : 0.f;
    return LLVQ_OK;
}

thread_local std::string g_last_error;

int grid_for(const llvq_codec *c, long long work, int threads) {
    long long want = (work + threads - 1) / threads;
    long long cap = (long long)c->num_sms * 3;
    return (int)std::max(1LL, std::min(want, cap));
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

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

template <int B>
cudaError_t launch_gemm48(const llvq_codec *c, const llvq_weight *w, const void *X, float *Y,
                          cudaStream_t st) {
    const int threads = 512;
    int grid = c->num_sms * gemm_ctas_per_sm<B>();
    int rpc = std::max((w->rows + grid - 1) / grid, 1);
    grid = (w->rows + rpc - 1) / rpc;
    const size_t smem = sizeof(Smem48) + (size_t)B * rpc * 32 * sizeof(float);
    const int nb = w->blocks_per_row;
    // block index -> row by a multiply-high: exact while rpc * nb < 2^32 / nb
    if ((unsigned long long)rpc * nb * nb >= (1ull << 32)) return cudaErrorInvalidValue;
    const uint32_t recip = nb > 1 ? (uint32_t)(((1ull << 32) + nb - 1) / nb) : 0u;
    static bool attr_set[17] = {false};
    if (!attr_set[B]) {
        cudaFuncSetAttribute(k_gemm48<B>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        attr_set[B] = true;
    }
    if (smem > 200 * 1024) return cudaErrorInvalidValue;
    k_gemm48<B><<<grid, threads, smem, st>>>(c->d_image48, (int)c->nclasses,
                                             (unsigned long long)c->npoints,
                                             (const unsigned long long *)w->words, w->row_pitch_words,
                                             w->rows, nb, recip, w->gain_mode,
                                             (const __half_raw *)w->gains, (const __half_raw *)X, Y, rpc,
                                             c->d_flags);
    return cudaGetLastError();
}

}  // namespace

extern "C" {

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
    if (index_bits != 48) return LLVQ_ERR_UNSUPPORTED;
    HostTables T;
    std::string err;
    if (!build_host_tables(index_bits, T, err)) { g_last_error = err; return LLVQ_ERR_UNSUPPORTED; }
    std::vector<unsigned char> buf(sizeof(Smem48));
    Smem48 &S = *reinterpret_cast<Smem48 *>(buf.data());
    llvq_status st = build_image48(T, S, err);
    if (st != LLVQ_OK) { g_last_error = err; return st; }
    llvq_codec *c = new llvq_codec;
    c->index_bits = index_bits;
    c->M = T.M;
    c->npoints = T.n_points;
    c->nclasses = (int64_t)T.classes.size();
    if (cudaGetDevice(&c->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess ||
        cudaMalloc(&c->d_image48, sizeof(Smem48)) != cudaSuccess ||
        cudaMemcpy(c->d_image48, buf.data(), sizeof(Smem48), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMalloc(&c->d_flags, sizeof(unsigned)) != cudaSuccess ||
        cudaMemset(c->d_flags, 0, sizeof(unsigned)) != cudaSuccess) {
        cudaGetLastError();
        llvq_codec_destroy(c);
        return LLVQ_ERR_CUDA;
    }
    static std::once_flag once;
    std::call_once(once, [] {
        cudaFuncSetAttribute(k_decode48, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem48));
    });
    *out = c;
    return LLVQ_OK;
}

void llvq_codec_destroy(llvq_codec *c) {
    if (!c) return;
    if (c->d_image48) cudaFree(c->d_image48);
    if (c->d_flags) cudaFree(c->d_flags);
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
    const int threads = 512;
    const int grid = grid_for(c, n, threads);
    k_decode48<<<grid, threads, sizeof(Smem48), st>>>(c->d_image48, (int)c->nclasses,
                                                       (unsigned long long)c->npoints,
                                                       (const unsigned long long *)d_words, n, d_out,
                                                       c->d_flags);
    return cudaGetLastError() == cudaSuccess ? LLVQ_OK : LLVQ_ERR_CUDA;
}

llvq_status llvq_gemm_smallbatch(const llvq_codec *c, const llvq_weight *w, const void *d_X,
                                 int32_t batch, float *d_Y, void *stream) {
    if (!c) return LLVQ_ERR_ARG;
    llvq_status st = check_weight(c, w);
    if (st != LLVQ_OK) return st;
    if (batch < 1 || batch > 16 || !d_X || !d_Y) return LLVQ_ERR_ARG;
    if (!aligned(d_X, 16) || !aligned(d_Y, 4)) return LLVQ_ERR_ARG;
    if (w->rows == 0) return LLVQ_OK;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    switch (batch) {
        case 1: e = launch_gemm48<1>(c, w, d_X, d_Y, s); break;
        case 2: e = launch_gemm48<2>(c, w, d_X, d_Y, s); break;
        case 3: e = launch_gemm48<3>(c, w, d_X, d_Y, s); break;
        case 4: e = launch_gemm48<4>(c, w, d_X, d_Y, s); break;
        case 5: e = launch_gemm48<5>(c, w, d_X, d_Y, s); break;
        case 6: e = launch_gemm48<6>(c, w, d_X, d_Y, s); break;
        case 7: e = launch_gemm48<7>(c, w, d_X, d_Y, s); break;
        case 8: e = launch_gemm48<8>(c, w, d_X, d_Y, s); break;
        case 9: e = launch_gemm48<9>(c, w, d_X, d_Y, s); break;
        case 10: e = launch_gemm48<10>(c, w, d_X, d_Y, s); break;
        case 11: e = launch_gemm48<11>(c, w, d_X, d_Y, s); break;
        case 12: e = launch_gemm48<12>(c, w, d_X, d_Y, s); break;
        case 13: e = launch_gemm48<13>(c, w, d_X, d_Y, s); break;
        case 14: e = launch_gemm48<14>(c, w, d_X, d_Y, s); break;
        case 15: e = launch_gemm48<15>(c, w, d_X, d_Y, s); break;
        default: e = launch_gemm48<16>(c, w, d_X, d_Y, s); break;
    }
    return e == cudaSuccess ? LLVQ_OK : LLVQ_ERR_CUDA;
}

llvq_status llvq_gemv(const llvq_codec *c, const llvq_weight *w, const void *d_x, float *d_y,
                      void *stream) {
    return llvq_gemm_smallbatch(c, w, d_x, 1, d_y, stream);
}

llvq_status llvq_get_error(const llvq_codec *c, void *stream, uint32_t *flags) {
    if (!c || !flags) return LLVQ_ERR_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned h = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess ||
        cudaMemcpy(&h, c->d_flags, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(c->d_flags, 0, sizeof(unsigned)) != cudaSuccess) {
        return LLVQ_ERR_CUDA;
    }
    *flags = h;
    return h ? LLVQ_ERR_DEVICE_FLAG : LLVQ_OK;
}

}  // extern "C"
