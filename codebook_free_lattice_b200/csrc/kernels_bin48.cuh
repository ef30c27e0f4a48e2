// kernels_bin48.cuh -- 48-bit decode and fused decode-and-multiply with the blocks sorted by coset.
//
// "Leech Lattice Vector Quantization for Efficient LLM Compression", papernotes.org notes,
// 方法详解 / 关键设计 2 and 4: every block is decoded to its 24-dim integer vector in registers
// and multiplied with the activations; dequantized weights never reach global memory.
//
// The arrangement decode of an odd-coset block (one coordinate set) and of an even-coset block
// (two coordinate sets) are different instruction streams; a warp holding both kinds would run
// both.  So each CTA works in chunks: phase 1 classifies the chunk's blocks (class, digits r, s,
// p) and writes a 16-byte record per block into a shared-memory list, odd-coset records from the
// front and even-coset records from the back; in phase 2 every warp takes 32 records of one list
// at a time, so each warp runs one decode path.  The next chunk's packed words load during
// phase 2.  One kernel body serves two outputs (sinks): the fused product (GemvSink; short row
// ranges, see kernels_gemv48.cuh for the long ones) and the plain decode to int8 vectors
// (DecodeSink).
#pragma once
#include "kernels.cuh"

namespace llvq {

constexpr int kBinThreads = 1024;                 // one CTA per SM, 64 registers per thread
constexpr int kBinPer = 5;                        // blocks per thread and chunk (80 KB of records)
// A CTA splits its blocks into equal chunks of at most PER blocks per thread, so that no chunk is
// a small remainder.

// One classified block.  y = class | r << 9 | (see below) << 21; z = s | gain code << 24;
// w = the sink's position of the block.  Odd classes and even classes off the table path:
// x = p bits 0..31, y bit 21 = p bit 32.  Even classes on the table path: x = the complement's
// code sequence (fetched while classifying), y bits 21..31 = p_S.
using BinRec = uint4;

// shared memory of a binned kernel: tables, records, counters and mbarrier, then the sink's own
__host__ __device__ constexpr size_t bin48_base_smem(int per) {
    return sizeof(Smem48) + sizeof(SmemEven48) + sizeof(BinRec) * kBinThreads * per + 8 * sizeof(int) + 8;
}
__host__ __device__ constexpr size_t bin48_smem_bytes(int batch, int rows_per_cta, int per) {
    return bin48_base_smem(per) + sizeof(float) * (size_t)batch * rows_per_cta * 32;
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

// Fused product: a CTA owns rows [row0, row0 + rows_per_cta); block t of the CTA is row t / nb
// (multiply-high with ceil(2^32 / nb)), column t mod nb; record position = row | column << 16.
template <int BATCH>
struct GemvSink {
    const unsigned long long *words;
    long long pitch;
    int rows, nb;
    uint32_t nb_recip;
    int gain_mode;
    const __half *gains, *X;
    float *Y;
    int rows_per_cta;
    // per CTA
    int row0, nrows;
    float *acc;

    __device__ void init(unsigned char *extra) {
        acc = reinterpret_cast<float *>(extra);                 // [BATCH][rows_per_cta][32]
        for (int i = threadIdx.x; i < BATCH * rows_per_cta * 32; i += kBinThreads) acc[i] = 0.f;
        row0 = blockIdx.x * rows_per_cta;
        nrows = max(0, min(rows_per_cta, rows - row0));
    }
    __device__ int total() const { return nrows * nb; }
    __device__ int row_of(int t) const { return nb == 1 ? t : (int)__umulhi((uint32_t)t, nb_recip); }
    __device__ unsigned long long load(int t) const {
        const int rl = row_of(t);
        return __ldg(words + (long long)(row0 + rl) * pitch + (t - rl * nb));
    }
    __device__ uint32_t where(int t) const {
        const int rl = row_of(t);
        return (uint32_t)rl | (uint32_t)(t - rl * nb) << 16;
    }
    __device__ void invalid(int) const {}                       // a bad index contributes nothing
    __device__ void consume(const uint32_t v[6], uint32_t info, uint32_t z, uint32_t w, const Smem48 &S,
                            int lane) const {
        const int rl = (int)(w & 0xFFFFu), j = (int)(w >> 16);
        const long long row = (long long)row0 + rl;
        const float scale = gain_mode == 0 ? __half2float(__ldg(gains + row * nb + j))
                                           : __half2float(__ldg(gains + row * 256 + (z >> 24))) *
                                                 S.invnorm[info_m(info)];
        accumulate_block<BATCH>(v, scale, X, (long long)nb * 24, j, acc, rl, rows_per_cta, lane);
    }
    __device__ void finish(int lane) const {
        const int warp = threadIdx.x >> 5;
        for (int i = warp; i < BATCH * nrows; i += kBinThreads >> 5) {
            const int bb = i / nrows, rl = i - bb * nrows;
            float sum = acc[(bb * rows_per_cta + rl) * 32 + lane];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
            if (lane == 0) Y[(long long)bb * rows + row0 + rl] = sum;
        }
    }
};

// Plain decode: a CTA owns words [base, base + per_cta); record position = t; output int8 [n][24].
struct DecodeSink {
    const unsigned long long *words;
    long long n;
    int8_t *out;
    long long per_cta;
    // per CTA
    long long base;
    int count;

    __device__ void init(unsigned char *) {
        base = (long long)blockIdx.x * per_cta;
        count = (int)max(0LL, min(per_cta, n - base));
    }
    __device__ int total() const { return count; }
    __device__ unsigned long long load(int t) const { return __ldg(words + base + t); }
    __device__ uint32_t where(int t) const { return (uint32_t)t; }
    __device__ void store(int t, const uint32_t v[6]) const {
        uint2 *o = reinterpret_cast<uint2 *>(out + (base + t) * 24);
        o[0] = make_uint2(v[0], v[1]);
        o[1] = make_uint2(v[2], v[3]);
        o[2] = make_uint2(v[4], v[5]);
    }
    __device__ void invalid(int t) const {                       // a bad index decodes to zero
        const uint32_t z[6] = {0u, 0u, 0u, 0u, 0u, 0u};
        store(t, z);
    }
    __device__ void consume(const uint32_t v[6], uint32_t, uint32_t, uint32_t w, const Smem48 &, int) const {
        store((int)w, v);
    }
    __device__ void finish(int) const {}
};

// The generic decode for the rare even classes off the table path, kept out of line so that it
// does not raise the register count of the common paths.
__device__ __noinline__ void arrange48_rare(const Smem48 &S, int cls, uint32_t info, unsigned long long p,
                                            uint32_t r, uint32_t s, uint32_t *v) {
    arrange48(S, cls, info, p, r, s, true, v);
}

// Phase 2 for one record of the coset ODD.
template <bool ODD, class Sink>
__device__ __forceinline__ void bin48_process(const BinRec e, const Smem48 &S, const SmemEven48 &E,
                                              const Sink &sink, int lane) {
    const int cls = (int)(e.y & 0x1FFu);
    const uint32_t r = (e.y >> 9) & 0xFFFu;
    const uint32_t s = e.z & 0xFFFFFFu;
    const uint32_t info = S.c_info[cls];
    const unsigned long long p = (unsigned long long)((e.y >> 21) & 1u) << 32 | e.x;
    uint32_t v[6];
    if (ODD) arrange_odd48(S, cls, info, p, r, v);
    else if (info & kInfoTable)
        even48_merge(S, E, info, S.c_info2[cls], r, s, E.tabS[(S.c_offs[cls] >> 19) + (e.y >> 21)], e.x, v);
    else arrange48_rare(S, cls, info, p, r, s, v);
    sink.consume(v, info, e.z, e.w, S, lane);
}

template <class Sink, int PER>
__global__ void __launch_bounds__(kBinThreads, 1) k_bin48(Dec48::Args args, const SmemEven48 *even,
                                                          const uint32_t *__restrict__ tabC, Sink sink,
                                                          unsigned *__restrict__ flags, uint32_t wait_tries) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem48 &S = *reinterpret_cast<Smem48 *>(smem_raw);
    SmemEven48 &E = *reinterpret_cast<SmemEven48 *>(smem_raw + sizeof(Smem48));
    BinRec *list = reinterpret_cast<BinRec *>(smem_raw + sizeof(Smem48) + sizeof(SmemEven48));
    constexpr int kCap = kBinThreads * PER;                                 // records per chunk
    // [2 chunk parities][odd count | even count << 16, -, odd taken, even taken]
    int *counts = reinterpret_cast<int *>(list + kCap);
    unsigned long long *bar = reinterpret_cast<unsigned long long *>(counts + 8);   // 8-byte aligned
    sink.init(smem_raw + bin48_base_smem(PER));
    if (threadIdx.x < 8) counts[threadIdx.x] = 0;
    const int total = sink.total();
    const int nchunks = (total + kCap - 1) / kCap;
    const int chunk = nchunks > 0 ? (total + nchunks - 1) / nchunks : 0;
    const int lane = threadIdx.x & 31;
    const unsigned lanes_below = (1u << lane) - 1u;
    const int warp_t0 = threadIdx.x & ~31;
    bool bad = false;

    unsigned long long wnext[PER];
#pragma unroll
    for (int k = 0; k < PER; k++) {
        const int t = k * kBinThreads + threadIdx.x;
        wnext[k] = t < min(chunk, total) ? sink.load(t) : 0ull;
    }
    {
        void *const dst[2] = {&S, &E};
        const void *const src[2] = {args.image, even};
        const uint32_t bytes[2] = {(uint32_t)sizeof(Smem48), (uint32_t)sizeof(SmemEven48)};
        if (!bulk_load_smem(dst, src, bytes, bar, wait_tries)) {
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
        // phase 1: classify this thread's blocks of the chunk and append each record to its list
        // (one packed shared-memory atomic per warp and block slot reserves the places in both
        // lists); an even block on the table path carries its complement code sequence
#pragma unroll
        for (int k = 0; k < PER; k++) {
            if (base + k * kBinThreads + warp_t0 >= end) break;              // warp-uniform
            const int t = base + k * kBinThreads + threadIdx.x;
            const Cls48 c = classify48(wnext[k], S, args.npoints);
            const bool valid = t < end;
            if (valid && !c.ok) {
                bad = true;
                sink.invalid(t);
            }
            const bool enq = valid && c.ok;
            const bool odd = c.info & kInfoOdd;
            BinRec rec;
            rec.z = c.s | (uint32_t)((wnext[k] >> 48) & 0xFFu) << 24;
            if (!odd && (c.info & kInfoTable)) {
                const Even48Idx ix = even48_indices(S, c.cls, c.p);
                rec.x = enq ? __ldg(tabC + (S.c_offs[c.cls] & 0x7FFFFu) + ix.pC) : 0u;
                rec.y = (uint32_t)c.cls | c.r << 9 | ix.pS << 21;
            } else {
                rec.x = (uint32_t)c.p;
                rec.y = (uint32_t)c.cls | c.r << 9 | (uint32_t)(c.p >> 32) << 21;
            }
            const unsigned mo = __ballot_sync(0xFFFFFFFFu, enq && odd);
            const unsigned me = __ballot_sync(0xFFFFFFFFu, enq && !odd);
            uint32_t b0 = 0;
            if (lane == 0 && (mo | me)) b0 = atomicAdd(reinterpret_cast<unsigned *>(cnt), __popc(mo) | __popc(me) << 16);
            b0 = __shfl_sync(0xFFFFFFFFu, b0, 0);
            if (enq) {
                rec.w = sink.where(t);
                const int pos = odd ? (int)((b0 & 0xFFFFu) + __popc(mo & lanes_below))
                                    : kCap - 1 - (int)((b0 >> 16) + __popc(me & lanes_below));
                list[pos] = rec;
            }
        }
        // the next chunk's words load while this chunk decodes
#pragma unroll
        for (int k = 0; k < PER; k++) {
            const int t = end + k * kBinThreads + threadIdx.x;
            wnext[k] = t < min(end + chunk, total) ? sink.load(t) : 0ull;
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
                    if (list_id == 0) bin48_process<true>(list[i], S, E, sink, lane);
                    else bin48_process<false>(list[kCap - 1 - i], S, E, sink, lane);
                }
            }
        }
    }
    __syncthreads();
    sink.finish(lane);
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicOr(flags, kFlagIndexRange);
}

}  // namespace llvq
