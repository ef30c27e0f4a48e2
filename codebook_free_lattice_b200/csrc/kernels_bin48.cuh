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
// A chunk holds up to PER blocks per thread (PER = 4 or 5: 64 or 80 KB of records); a CTA splits
// its blocks into equal chunks so that no chunk is a small remainder.

// One classified block.  y = class | r << 9 | (see below) << 21; z = s | gain code << 24;
// w = row within the CTA | block column j << 16.  Odd classes and even classes off the table
// path: x = p bits 0..31, y bit 21 = p bit 32.  Even classes on the table path: x = the
// complement's code sequence (fetched while classifying), y bits 21..31 = p_S.
using BinRec = uint4;

__host__ __device__ constexpr size_t bin48_smem_bytes(int batch, int rows_per_cta, int per) {
    return sizeof(Smem48) + sizeof(SmemEven48) + sizeof(BinRec) * kBinThreads * per +
           sizeof(float) * (size_t)batch * rows_per_cta * 32 + 8 * sizeof(int) + 8;
}

// y contribution of one decoded block: scale * <v, x_b> for every batch row b, added to the
// CTA's shared accumulators (slot per lane; warps of the CTA may meet on a slot).
template <int BATCH>
__device__ __forceinline__ void accumulate_block(const uint32_t v[6], float scale, const __half *__restrict__ X,
                                                 long long K, int j, float *acc, int rl, int rows_per_cta,
                                                 int lane) {
    uint32_t wh[12];                                           // exact fp16 coordinates, in pairs
#pragma unroll
    for (int q = 0; q < 6; q++) i8x4_to_h2x2(v[q], wh[2 * q], wh[2 * q + 1]);
#pragma unroll
    for (int bb = 0; bb < BATCH; bb++) {
        const uint4 *xp = reinterpret_cast<const uint4 *>(X + bb * K + (long long)j * 24);
        float d0 = 0.f, d1 = 0.f;                              // two chains for latency
#pragma unroll
        for (int c = 0; c < 3; c++) {
            const uint4 raw = __ldg(xp + c);
            d0 = fma2_f16_f32(wh[4 * c + 0], raw.x, d0);
            d1 = fma2_f16_f32(wh[4 * c + 1], raw.y, d1);
            d0 = fma2_f16_f32(wh[4 * c + 2], raw.z, d0);
            d1 = fma2_f16_f32(wh[4 * c + 3], raw.w, d1);
        }
        atomicAdd(&acc[(bb * rows_per_cta + rl) * 32 + lane], scale * (d0 + d1));
    }
}

// Phase 2 for one record of the coset ODD.
template <bool ODD, int BATCH>
__device__ __forceinline__ void bin48_process(const BinRec e, const Smem48 &S, const SmemEven48 &E, int gain_mode,
                                              const __half *__restrict__ gains, const __half *__restrict__ X,
                                              long long K, int row0, int nb, float *acc, int rows_per_cta,
                                              int lane) {
    const int cls = (int)(e.y & 0x1FFu);
    const uint32_t r = (e.y >> 9) & 0xFFFu;
    const uint32_t s = e.z & 0xFFFFFFu;
    const int code = (int)(e.z >> 24);
    const int rl = (int)(e.w & 0xFFFFu);
    const int j = (int)(e.w >> 16);
    const uint32_t info = S.c_info[cls];
    const unsigned long long p = (unsigned long long)((e.y >> 21) & 1u) << 32 | e.x;
    uint32_t v[6];
    if (ODD) arrange_odd48(S, cls, info, p, r, v);
    else if (info & kInfoTable)
        even48_merge(S, E, info, S.c_info2[cls], r, s, E.tabS[(S.c_offs[cls] >> 19) + (e.y >> 21)], e.x, v);
    else arrange48(S, cls, info, p, r, s, true, v);
    const long long row = (long long)row0 + rl;
    const float scale = gain_mode == 0 ? __half2float(__ldg(gains + row * nb + j))
                                       : __half2float(__ldg(gains + row * 256 + code)) * S.invnorm[info_m(info)];
    accumulate_block<BATCH>(v, scale, X, K, j, acc, rl, rows_per_cta, lane);
}

template <int BATCH, int PER>
__global__ void __launch_bounds__(kBinThreads, 1) k_gemm_bin48(
    Dec48::Args args, const SmemEven48 *even, const uint32_t *__restrict__ tabC,
    const unsigned long long *__restrict__ words, long long pitch, int rows, int nb,
    uint32_t nb_recip, int gain_mode, const __half *__restrict__ gains, const __half *__restrict__ X,
    float *__restrict__ Y, int rows_per_cta, unsigned *__restrict__ flags) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem48 &S = *reinterpret_cast<Smem48 *>(smem_raw);
    SmemEven48 &E = *reinterpret_cast<SmemEven48 *>(smem_raw + sizeof(Smem48));
    BinRec *list = reinterpret_cast<BinRec *>(smem_raw + sizeof(Smem48) + sizeof(SmemEven48));
    constexpr int kCap = kBinThreads * PER;                                 // records per chunk
    float *acc = reinterpret_cast<float *>(list + kCap);                    // [BATCH][rows_per_cta][32]
    // [2 chunk parities][odd count | even count << 16, -, odd taken, even taken]
    int *counts = reinterpret_cast<int *>(acc + BATCH * rows_per_cta * 32);
    unsigned long long *bar = reinterpret_cast<unsigned long long *>(counts + 8);   // 8-byte aligned
    for (int i = threadIdx.x; i < BATCH * rows_per_cta * 32; i += kBinThreads) acc[i] = 0.f;
    if (threadIdx.x < 8) counts[threadIdx.x] = 0;
    const int row0 = blockIdx.x * rows_per_cta;
    const int nrows = max(0, min(rows_per_cta, rows - row0));
    const int total = nrows * nb;
    const int nchunks = (total + kCap - 1) / kCap;
    const int chunk = nchunks > 0 ? (total + nchunks - 1) / nchunks : 0;
    const long long K = (long long)nb * 24;
    const int lane = threadIdx.x & 31;
    const unsigned lanes_below = (1u << lane) - 1u;
    bool bad = false;

    // block t of the CTA -> row rl = t / nb (multiply-high with ceil(2^32 / nb)), column t - rl nb
    const unsigned long long *wbase = words + (long long)row0 * pitch;
    const int warp_t0 = threadIdx.x & ~31;
    unsigned long long wnext[PER];
#pragma unroll
    for (int k = 0; k < PER; k++) {
        const int t = k * kBinThreads + threadIdx.x;
        const int rl = nb == 1 ? t : (int)__umulhi((uint32_t)t, nb_recip);
        wnext[k] = t < min(chunk, total) ? __ldg(wbase + (long long)rl * pitch + (t - rl * nb)) : 0ull;
    }
    {
        void *const dst[2] = {&S, &E};
        const void *const src[2] = {args.image, even};
        const uint32_t bytes[2] = {(uint32_t)sizeof(Smem48), (uint32_t)sizeof(SmemEven48)};
        if (!bulk_load_smem(dst, src, bytes, bar)) {
            if (threadIdx.x == 0) atomicOr(flags, kFlagWaitTimeout);
            return;
        }
    }
    int parity = 0;
    for (int base = 0; base < total; base += chunk, parity ^= 1) {
        const int end = min(base + chunk, total);
        __syncthreads();                       // previous chunk's records consumed; counts reset
        int *cnt = counts + 4 * parity;
        if (threadIdx.x < 4) counts[4 * (parity ^ 1) + threadIdx.x] = 0;
        // phase 1a: classify this thread's blocks of the chunk; an even block on the table path
        // starts the fetch of its complement code sequence (global memory) right away
        BinRec rec[PER];
        bool enq[PER], odd[PER];
#pragma unroll
        for (int k = 0; k < PER; k++) {
            const int t = base + k * kBinThreads + threadIdx.x;
            enq[k] = false;
            odd[k] = false;
            if (base + k * kBinThreads + warp_t0 >= end) continue;           // warp-uniform
            const Cls48 c = classify48(wnext[k], S, args.npoints);
            const bool valid = t < end;
            bad |= valid && !c.ok;
            enq[k] = valid && c.ok;
            odd[k] = c.info & kInfoOdd;
            rec[k].z = c.s;
            if (!odd[k] && (c.info & kInfoTable)) {
                const Even48Idx ix = even48_indices(S, c.cls, c.p);
                rec[k].x = enq[k] ? __ldg(tabC + (S.c_offs[c.cls] & 0x7FFFFu) + ix.pC) : 0u;
                rec[k].y = (uint32_t)c.cls | c.r << 9 | ix.pS << 21;
            } else {
                rec[k].x = (uint32_t)c.p;
                rec[k].y = (uint32_t)c.cls | c.r << 9 | (uint32_t)(c.p >> 32) << 21;
            }
        }
        // phase 1b: one shared-memory atomic per warp reserves its places in both lists
        {
            unsigned mo[PER], me[PER];
            uint32_t no_w = 0, ne_w = 0;
#pragma unroll
            for (int k = 0; k < PER; k++) {
                mo[k] = __ballot_sync(0xFFFFFFFFu, enq[k] && odd[k]);
                me[k] = __ballot_sync(0xFFFFFFFFu, enq[k] && !odd[k]);
                no_w += __popc(mo[k]);
                ne_w += __popc(me[k]);
            }
            uint32_t b0 = 0;
            if (lane == 0 && (no_w | ne_w)) b0 = atomicAdd(reinterpret_cast<unsigned *>(cnt), no_w | ne_w << 16);
            b0 = __shfl_sync(0xFFFFFFFFu, b0, 0);
            uint32_t bo = b0 & 0xFFFFu, be = b0 >> 16;
#pragma unroll
            for (int k = 0; k < PER; k++) {
                if (enq[k]) {
                    const int t = base + k * kBinThreads + threadIdx.x;
                    const int rl = nb == 1 ? t : (int)__umulhi((uint32_t)t, nb_recip);
                    rec[k].z |= (uint32_t)((wnext[k] >> 48) & 0xFFu) << 24;
                    rec[k].w = (uint32_t)rl | (uint32_t)(t - rl * nb) << 16;
                    const int pos = odd[k] ? (int)(bo + __popc(mo[k] & lanes_below))
                                           : kCap - 1 - (int)(be + __popc(me[k] & lanes_below));
                    list[pos] = rec[k];
                }
                bo += __popc(mo[k]);
                be += __popc(me[k]);
            }
        }
        // the next chunk's words load while this chunk decodes
#pragma unroll
        for (int k = 0; k < PER; k++) {
            const int t = end + k * kBinThreads + threadIdx.x;
            const int rl = nb == 1 ? t : (int)__umulhi((uint32_t)t, nb_recip);
            wnext[k] = t < min(end + chunk, total) ? __ldg(wbase + (long long)rl * pitch + (t - rl * nb)) : 0ull;
        }
        __syncthreads();
        // phase 2: each warp takes the next 32 records of a list until both lists are used up;
        // even-numbered warps start on the odd-coset list and odd-numbered warps on the even-coset
        // list, so the arithmetic-heavy and the lookup-latency-bound decodes share the SM
        const int first = (threadIdx.x >> 5) & 1;
        for (int pass = 0; pass < 2; pass++) {
            const int list_id = first ^ pass;
            const int n = list_id == 0 ? (cnt[0] & 0xFFFF) : (cnt[0] >> 16);
            while (true) {
                int i0 = 0;
                if (lane == 0) i0 = atomicAdd(cnt + 2 + list_id, 32);
                i0 = __shfl_sync(0xFFFFFFFFu, i0, 0);
                if (i0 >= n) break;
                const int i = i0 + lane;
                if (i < n) {
                    if (list_id == 0)
                        bin48_process<true, BATCH>(list[i], S, E, gain_mode, gains, X, K, row0, nb, acc,
                                                   rows_per_cta, lane);
                    else
                        bin48_process<false, BATCH>(list[kCap - 1 - i], S, E, gain_mode, gains, X, K,
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
