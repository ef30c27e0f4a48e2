// kernels_bin48.cuh -- fused decode-and-multiply at 48 bits with the blocks sorted by coset.
//
// "Leech Lattice Vector Quantization for Efficient LLM Compression", papernotes.org notes,
// 方法详解 / 关键设计 2 and 4: every block is decoded to its 24-dim integer vector in registers
// and multiplied with the activations; dequantized weights never reach global memory.
//
// The arrangement decode of an odd-coset block (one coordinate set) and of an even-coset block
// (two coordinate sets) are different instruction streams; a warp holding both kinds would run
// both.  So each CTA works in chunks: phase 1 classifies the chunk's blocks (class, digits r, s,
// p) and writes a 16-byte record per block into a shared-memory list, odd-coset records from the
// front and even-coset records from the back; phase 2 decodes the odd records, then the even
// ones, with every warp on one path.  The next chunk's packed words are loaded during phase 2.
#pragma once
#include "kernels.cuh"

namespace llvq {

constexpr int kBinThreads = 1024;                 // one CTA per SM, 64 registers per thread
constexpr int kBinPer = 4;                        // blocks per thread and chunk
constexpr int kBinChunk = kBinThreads * kBinPer;  // 4096 blocks = 64 KB of records

// One classified block: x = p bits 0..31; y = p bit 32 | class << 1 | r << 10 | gain code << 22;
// z = s; w = row within the CTA | block column j << 16.
using BinRec = uint4;

__host__ __device__ constexpr size_t bin48_smem_bytes(int batch, int rows_per_cta) {
    return sizeof(Smem48) + sizeof(SmemEven48) + sizeof(BinRec) * kBinChunk +
           sizeof(float) * (size_t)batch * rows_per_cta * 32 + 8 * sizeof(int);
}

// y contribution of one decoded block: scale * <v, x_b> for every batch row b, added to the
// CTA's shared accumulators (slot per lane; warps of the CTA may meet on a slot).
template <int BATCH>
__device__ __forceinline__ void accumulate_block(const uint32_t v[6], float scale, const __half *__restrict__ X,
                                                 long long K, int j, float *acc, int rl, int rows_per_cta,
                                                 int lane) {
    float wv[24];
#pragma unroll
    for (int q = 0; q < 6; q++)
#pragma unroll
        for (int e = 0; e < 4; e++) wv[4 * q + e] = (float)(int8_t)(v[q] >> (8 * e));
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
        atomicAdd(&acc[(bb * rows_per_cta + rl) * 32 + lane], scale * dot);
    }
}

struct BinFields {
    unsigned long long p;
    uint32_t r, s;
    int cls, code, rl, j;
};

__device__ __forceinline__ BinFields bin_unpack(const BinRec e) {
    BinFields f;
    f.p = (unsigned long long)(e.y & 1u) << 32 | e.x;
    f.cls = (int)((e.y >> 1) & 0x1FFu);
    f.r = (e.y >> 10) & 0xFFFu;
    f.code = (int)(e.y >> 22);
    f.s = e.z;
    f.rl = (int)(e.w & 0xFFFFu);
    f.j = (int)(e.w >> 16);
    return f;
}

// Phase 2 for one record of the coset ODD.
template <bool ODD, int BATCH>
__device__ __forceinline__ void bin48_process(const BinRec e, const Smem48 &S, const SmemEven48 &E,
                                              const uint32_t *__restrict__ tabC, int gain_mode,
                                              const __half *__restrict__ gains, const __half *__restrict__ X,
                                              long long K, int row0, int nb, float *acc, int rows_per_cta,
                                              int lane) {
    const BinFields f = bin_unpack(e);
    const uint32_t info = S.c_info[f.cls];
    uint32_t v[6];
    if (ODD) arrange_odd48(S, f.cls, info, f.p, f.r, v);
    else if (info & kInfoTable) arrange_even48_table(S, E, tabC, f.cls, info, f.p, f.r, f.s, v);
    else arrange48(S, f.cls, info, f.p, f.r, f.s, true, v);
    const long long row = (long long)row0 + f.rl;
    const float scale = gain_mode == 0 ? __half2float(__ldg(gains + row * nb + f.j))
                                       : __half2float(__ldg(gains + row * 256 + f.code)) * S.invnorm[info_m(info)];
    accumulate_block<BATCH>(v, scale, X, K, f.j, acc, f.rl, rows_per_cta, lane);
}

template <int BATCH>
__global__ void __launch_bounds__(kBinThreads, 1) k_gemm_bin48(
    Dec48::Args args, const SmemEven48 *even, const uint32_t *__restrict__ tabC,
    const unsigned long long *__restrict__ words, long long pitch, int rows, int nb,
    uint32_t nb_recip, int gain_mode, const __half *__restrict__ gains, const __half *__restrict__ X,
    float *__restrict__ Y, int rows_per_cta, unsigned *__restrict__ flags) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem48 &S = *reinterpret_cast<Smem48 *>(smem_raw);
    SmemEven48 &E = *reinterpret_cast<SmemEven48 *>(smem_raw + sizeof(Smem48));
    BinRec *list = reinterpret_cast<BinRec *>(smem_raw + sizeof(Smem48) + sizeof(SmemEven48));
    float *acc = reinterpret_cast<float *>(list + kBinChunk);              // [BATCH][rows_per_cta][32]
    // [2 chunk parities][odd count, even count, odd taken, even taken]
    int *counts = reinterpret_cast<int *>(acc + BATCH * rows_per_cta * 32);
    load_smem_image(&S, args.image, sizeof(Smem48));
    load_smem_image(&E, even, sizeof(SmemEven48));
    for (int i = threadIdx.x; i < BATCH * rows_per_cta * 32; i += kBinThreads) acc[i] = 0.f;
    if (threadIdx.x < 8) counts[threadIdx.x] = 0;
    const int row0 = blockIdx.x * rows_per_cta;
    const int nrows = max(0, min(rows_per_cta, rows - row0));
    const int total = nrows * nb;
    const long long K = (long long)nb * 24;
    const int lane = threadIdx.x & 31;
    const unsigned lanes_below = (1u << lane) - 1u;
    bool bad = false;

    // block t of the CTA -> row rl = t / nb (multiply-high with ceil(2^32 / nb)), column t - rl nb
    const unsigned long long *wbase = words + (long long)row0 * pitch;
    const int warp_t0 = threadIdx.x & ~31;
    unsigned long long wnext[kBinPer];
#pragma unroll
    for (int k = 0; k < kBinPer; k++) {
        const int t = k * kBinThreads + threadIdx.x;
        const int rl = nb == 1 ? t : (int)__umulhi((uint32_t)t, nb_recip);
        wnext[k] = t < total ? __ldg(wbase + (long long)rl * pitch + (t - rl * nb)) : 0ull;
    }
    int parity = 0;
    for (int base = 0; base < total; base += kBinChunk, parity ^= 1) {
        __syncthreads();                       // previous chunk's records consumed; counts reset
        int *cnt = counts + 4 * parity;
        if (threadIdx.x < 4) counts[4 * (parity ^ 1) + threadIdx.x] = 0;
        // phase 1: classify and sort by coset (warps past the end skip)
#pragma unroll
        for (int k = 0; k < kBinPer; k++) {
            if (base + k * kBinThreads + warp_t0 >= total) break;
            const int t = base + k * kBinThreads + threadIdx.x;
            const bool valid = t < total;
            const Cls48 c = classify48(wnext[k], S, args.npoints);
            bad |= valid && !c.ok;
            const bool enq = valid && c.ok;
            const bool odd = c.info & kInfoOdd;
            const unsigned mo = __ballot_sync(0xFFFFFFFFu, enq && odd);
            const unsigned me = __ballot_sync(0xFFFFFFFFu, enq && !odd);
            int bo = 0, be = 0;
            if (lane == 0) {
                if (mo) bo = atomicAdd(cnt, __popc(mo));
                if (me) be = atomicAdd(cnt + 1, __popc(me));
            }
            bo = __shfl_sync(0xFFFFFFFFu, bo, 0);
            be = __shfl_sync(0xFFFFFFFFu, be, 0);
            if (enq && !odd && (c.info & kInfoTable))   // complement table entry into L1 for phase 2
                asm volatile("prefetch.global.L1 [%0];" ::"l"(even48_tabC_entry(S, tabC, c.cls, c.p)));
            if (enq) {
                const int rl = nb == 1 ? t : (int)__umulhi((uint32_t)t, nb_recip);
                const int j = t - rl * nb;
                BinRec e;
                e.x = (uint32_t)c.p;
                e.y = (uint32_t)(c.p >> 32) | (uint32_t)c.cls << 1 | c.r << 10 |
                      (uint32_t)((wnext[k] >> 48) & 0xFFu) << 22;
                e.z = c.s;
                e.w = (uint32_t)rl | (uint32_t)j << 16;
                const int pos = odd ? bo + __popc(mo & lanes_below)
                                    : kBinChunk - 1 - (be + __popc(me & lanes_below));
                list[pos] = e;
            }
        }
        // the next chunk's words load while this chunk decodes
#pragma unroll
        for (int k = 0; k < kBinPer; k++) {
            const int t = base + kBinChunk + k * kBinThreads + threadIdx.x;
            const int rl = nb == 1 ? t : (int)__umulhi((uint32_t)t, nb_recip);
            wnext[k] = t < total ? __ldg(wbase + (long long)rl * pitch + (t - rl * nb)) : 0ull;
        }
        __syncthreads();
        const int no = cnt[0], ne = cnt[1];
        // phase 2: odd-coset records, then even-coset records; each warp takes the next 32
        // records of a list until both are used up
        for (int list_id = 0; list_id < 2; list_id++) {
            const int n = cnt[list_id];
            while (true) {
                int i0 = 0;
                if (lane == 0) i0 = atomicAdd(cnt + 2 + list_id, 32);
                i0 = __shfl_sync(0xFFFFFFFFu, i0, 0);
                if (i0 >= n) break;
                const int i = i0 + lane;
                if (i < n) {
                    if (list_id == 0)
                        bin48_process<true, BATCH>(list[i], S, E, tabC, gain_mode, gains, X, K, row0, nb, acc,
                                                   rows_per_cta, lane);
                    else
                        bin48_process<false, BATCH>(list[kBinChunk - 1 - i], S, E, tabC, gain_mode, gains, X, K,
                                                    row0, nb, acc, rows_per_cta, lane);
                }
            }
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    for (int i = warp; i < BATCH * nrows; i += kBinThreads >> 5) {
        const int bb = i / nrows, rl = i - bb * nrows;
        float sum = acc[(bb * rows_per_cta + rl) * 32 + lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        if (lane == 0) Y[(long long)bb * rows + row0 + rl] = sum;
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicOr(flags, kFlagIndexRange);
}

}  // namespace llvq
