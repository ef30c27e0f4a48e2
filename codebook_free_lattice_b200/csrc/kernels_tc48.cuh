// kernels_tc48.cuh -- 48-bit small-batch product on the tensor cores, with coset-sorted decode.
//
// "Leech Lattice Vector Quantization for Efficient LLM Compression", papernotes.org notes,
// 方法详解 / 关键设计 4 (the fused dequantize-and-multiply): decoded blocks never reach global
// memory; they are written as exact fp16 integers into a shared-memory A tile that feeds
// tcgen05.mma.
//
// A CTA (1024 threads, one per SM) owns a 128-row tile and a range of K rounds.  A round covers
// 8 blocks of each row (1024 blocks, one per thread to classify):
//   1. thread t classifies block (row t / 8, slot t % 8) and appends a record (with the block's
//      fp16 gain) to the odd or the even list, as in k_bin48; the next round's word, gain and
//      activation chunk are loaded meanwhile;
//   -- barrier --
//   2. the previous round's MMAs have had the whole classify phase to finish: a bounded wait on
//      their mbarrier, then warp w reads TMEM lanes 32 (w % 4).. (rows) and the 16 columns of
//      slot w / 4 and adds gain * D into its 16 fp32 accumulators (one per batch column);
//   3. the block-diagonal activation tiles B_0, B_1 (slots 0..3, 4..7; N = 4 slots x 16 batch
//      columns) are stored; warps take 32 records of one list at a time, decode them and write
//      the 24 exact fp16 values and the gain of each block to its A position (blocks outside
//      the matrix or with a bad index get a zero A entry and a zero gain);
//   -- barrier --
//   4. one thread issues 2 x 6 MMAs (M = 128, N = 64, K = 96) into 128 TMEM columns and commits
//      them to the mbarrier; the CTA goes on with the next round's classify at once.
// Two CTA barriers per round; the MMA round trip hides behind the classify phase.  At the end
// the 8 slots of each row are summed in shared memory and added into y (zeroed by the launch;
// K splits add).
#pragma once
#include "kernels_bin48.cuh"
#include "kernels_tc.cuh"

namespace llvq {

constexpr int kTc48Slots = 8;                             // blocks per row and round
constexpr int kTc48Threads = kTcRows * kTc48Slots;        // 1024
constexpr uint32_t kTc48TmemCols = 2 * kTcN;              // 128 fp32 columns

struct alignas(128) Tc48Smem {
    __align__(128) unsigned char A[2][kTcASize];          // slots 0..3 and 4..7; reused for row sums
    __align__(128) unsigned char B[2][kTcBSize];
    float gain[kTc48Slots][kTcRows];
    BinRec list[kTc48Threads];
    int counts[8];
    unsigned long long mbar_mma;
    unsigned long long mbar_load;
    uint32_t tmem_base;
    uint32_t status;
};
static_assert(kTcRows * 16 * sizeof(float) <= 2 * kTcASize, "row sums must fit in the A tiles");

// the tensor-core tiles start on a 128-byte boundary after the two table images
__host__ __device__ constexpr size_t tc48_tiles_offset() {
    return (sizeof(Smem48) + sizeof(SmemEven48) + 127) / 128 * 128;
}
__host__ __device__ constexpr size_t tc48_smem_bytes() { return tc48_tiles_offset() + sizeof(Tc48Smem); }

// exact fp16 pairs of one decoded block into its A position (slot jj, row dr)
__device__ __forceinline__ void tc48_store_a(Tc48Smem &T, int dr, int jj, const uint32_t v[6]) {
    uint32_t h[12];
#pragma unroll
    for (int q = 0; q < 6; q++) i8x4_to_h2x2(v[q], h[2 * q], h[2 * q + 1]);
    unsigned char *A = T.A[jj >> 2];
    const int j4 = jj & 3;
#pragma unroll
    for (int q = 0; q < 3; q++)
        *reinterpret_cast<uint4 *>(A + (3 * j4 + q) * kTcALbo + dr * 16) =
            make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
}

// bounded wait for the round's MMAs (at most `tries` polls); the result is the same in every lane
// of the warp, so the warp-collective TMEM load that follows is taken by all lanes or by none
constexpr uint32_t kMmaWaitTries = 1u << 20;
__device__ __forceinline__ bool tc48_wait_mma(Tc48Smem &T, uint32_t phase, uint32_t tries) {
    bool done = false;
    for (uint32_t it = 0; it < tries && !done; it++) done = mbar_try_wait_parity(smem_u32(&T.mbar_mma), phase);
    return __all_sync(0xFFFFFFFFu, done);
}

// gain * D of this warp's 32 rows and one slot (16 batch columns) into the accumulators
__device__ __forceinline__ void tc48_epilogue(uint32_t taddr, float g, float yacc[16]) {
    uint32_t d[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]), "=r"(d[6]), "=r"(d[7]),
          "=r"(d[8]), "=r"(d[9]), "=r"(d[10]), "=r"(d[11]), "=r"(d[12]), "=r"(d[13]), "=r"(d[14]), "=r"(d[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int b = 0; b < 16; b++) yacc[b] = fmaf(g, __uint_as_float(d[b]), yacc[b]);
}

__global__ void __launch_bounds__(kTc48Threads, 1) k_gemm_tc48(
    Dec48::Args args, const SmemEven48 *even, const uint32_t *__restrict__ tabC,
    const unsigned long long *__restrict__ words, long long pitch, int rows, int nb, int batch, int gain_mode,
    const __half *__restrict__ gains, const __half *__restrict__ X, float *__restrict__ Y, int rounds_per_split,
    unsigned *__restrict__ flags, uint32_t table_tries, uint32_t mma_tries) {
    extern __shared__ __align__(128) unsigned char smem_tc48[];
    Smem48 &S = *reinterpret_cast<Smem48 *>(smem_tc48);
    SmemEven48 &E = *reinterpret_cast<SmemEven48 *>(smem_tc48 + sizeof(Smem48));
    Tc48Smem &T = *reinterpret_cast<Tc48Smem *>(smem_tc48 + tc48_tiles_offset());
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const unsigned lanes_below = (1u << lane) - 1u;
    const int row0 = blockIdx.x * kTcRows;
    const int nrounds = (nb + kTc48Slots - 1) / kTc48Slots;
    const int c0 = blockIdx.y * rounds_per_split;
    const int c1 = min(c0 + rounds_per_split, nrounds);
    const long long K = (long long)nb * 24;
    const int dr = tid >> 3, djj = tid & 7;                   // classify role: row, slot
    const int row = row0 + dr;
    const bool row_in = row < rows;
    const unsigned short *gbits = reinterpret_cast<const unsigned short *>(gains);
    // activation role: threads 0..383 own one 16-byte chunk (slot, batch column, third) of B
    constexpr int kXChunks = kTcBlocks * 16 * 3;
    const bool xrole = tid < 2 * kXChunks;
    const int xhalf = tid / kXChunks, xu = tid % kXChunks;
    const int xq = xu % 3, xn = xu / 3;                       // n = 16 slot + b
    const int xjj = xn >> 4, xb = xn & 15;
    auto load_x = [&](int ch) {
        const int j = ch * kTc48Slots + 4 * xhalf + xjj;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (xrole && xb < batch && j < nb) v = __ldg(reinterpret_cast<const uint4 *>(X + xb * K + (long long)j * 24 + 8 * xq));
        return v;
    };
    // this thread's word (and, with per-block gains, its gain) of round ch
    auto load_word = [&](int ch) {
        const int j = ch * kTc48Slots + djj;
        return row_in && j < nb ? __ldg(words + (long long)row * pitch + j) : 0ull;
    };
    auto load_gain = [&](int ch) {
        const int j = ch * kTc48Slots + djj;
        return gain_mode == 0 && row_in && j < nb ? __ldg(gbits + (long long)row * nb + j) : (unsigned short)0;
    };

    // first round's word, gain and activations, then the tables (bulk copy, bounded wait)
    unsigned long long wcur = 0ull;
    unsigned short gcur = 0;
    if (c0 < c1) {
        wcur = load_word(c0);
        gcur = load_gain(c0);
    }
    if (tid < 8) T.counts[tid] = 0;
    // B tiles: only the diagonal chunks are written per round; the rest stays zero
    for (int i = tid; i < 2 * kTcBSize / 16; i += kTc48Threads)
        reinterpret_cast<uint4 *>(&T.B[0][0])[i] = make_uint4(0, 0, 0, 0);
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&T.mbar_mma)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        T.status = 0;
    }
    {
        void *const dst[2] = {&S, &E};
        const void *const src[2] = {args.image, even};
        const uint32_t bytes[2] = {(uint32_t)sizeof(Smem48), (uint32_t)sizeof(SmemEven48)};
        if (!bulk_load_smem(dst, src, bytes, &T.mbar_load, table_tries)) {
            if (tid == 0) atomicOr(flags, kFlagWaitTimeout);
            return;                                           // no TMEM allocated yet
        }
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&T.tmem_base)), "r"(kTc48TmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = T.tmem_base;

    const int lg = warp & 3, eslot = warp >> 2;               // epilogue role: lane quarter, slot
    const int em = lg * 32 + lane;
    const uint32_t etaddr = tmem + ((uint32_t)(lg * 32) << 16) + (uint32_t)(eslot * 16);
    float yacc[16];
#pragma unroll
    for (int b = 0; b < 16; b++) yacc[b] = 0.f;
    bool bad = false;
    uint32_t phase = 0;
    // committed MMAs not yet waited for by this warp, and their phase parity
    bool pending = false;
    uint32_t pphase = 0;

    for (int ch = c0; ch < c1; ch++) {
        const int j0 = ch * kTc48Slots;
        int *cnt = T.counts + 4 * (ch & 1);
        if (tid < 4) T.counts[4 * ((ch & 1) ^ 1) + tid] = 0;
        // the previous round's gain of this thread's epilogue row and slot (written before the
        // last barrier; this round's decode overwrites it only after the next one)
        const float gep = ch > c0 ? T.gain[eslot][em] : 0.f;
        // ---- 1. classify this thread's block; append its record
        bool zero_a;
        {
            const bool inside = row_in && j0 + djj < nb;
            const uint32_t code = (uint32_t)((wcur >> 48) & 0xFFu);
            const unsigned short gh = gain_mode == 0 ? gcur : inside ? __ldg(gbits + (long long)row * 256 + code) : (unsigned short)0;
            const Cls48 c = classify48(wcur, S, args.npoints);
            bad |= inside && !c.ok;
            const bool enq = inside && c.ok;
            const bool odd = c.info & kInfoOdd;
            zero_a = !enq;
            BinRec rec;
            rec.z = c.s | code << 24;
            rec.w = (uint32_t)dr | (uint32_t)djj << 8 | (uint32_t)gh << 16;
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
                const int pos = odd ? (int)((b0 & 0xFFFFu) + __popc(mo & lanes_below))
                                    : kTc48Threads - 1 - (int)((b0 >> 16) + __popc(me & lanes_below));
                T.list[pos] = rec;
            }
        }
        // the next round's word and gain load while this round decodes
        if (ch + 1 < c1) {
            wcur = load_word(ch + 1);
            gcur = load_gain(ch + 1);
        }
        __syncthreads();
        const uint4 xnow = load_x(ch);                          // L2-resident; lands during the wait
        // ---- 2. the previous round's products: bounded wait, then the epilogue
        if (ch > c0) {
            if (tc48_wait_mma(T, phase, mma_tries)) {
                pending = false;
                tc_fence_after();
                tc48_epilogue(etaddr, gep, yacc);
            } else if (lane == 0) {
                atomicOr(&T.status, 1u);
            }
            phase ^= 1u;
        }
        // ---- 3. this round's A and B tiles (the MMAs that read them have completed)
        if (zero_a) {
            const uint32_t z[6] = {0x0u, 0x0u, 0x0u, 0x0u, 0x0u, 0x0u};
            tc48_store_a(T, dr, djj, z);
            T.gain[djj][dr] = 0.f;
        }
        if (xrole) *reinterpret_cast<uint4 *>(T.B[xhalf] + (3 * xjj + xq) * kTcBLbo + xn * 16) = xnow;
        // decode the lists into A (odd-numbered warps start on the even list)
        const int first = warp & 1;
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
                    const BinRec e = list_id == 0 ? T.list[i] : T.list[kTc48Threads - 1 - i];
                    const int cls = (int)(e.y & 0x1FFu);
                    const uint32_t r = (e.y >> 9) & 0xFFFu, s = e.z & 0xFFFFFFu;
                    const uint32_t info = S.c_info[cls];
                    const unsigned long long p = (unsigned long long)((e.y >> 21) & 1u) << 32 | e.x;
                    uint32_t v[6];
                    if (list_id == 0) arrange_odd48(S, cls, info, p, r, v);
                    else if (info & kInfoTable)
                        even48_merge(S, E, info, S.c_info2[cls], r, s, E.tabS[(S.c_offs[cls] >> 19) + (e.y >> 21)],
                                     e.x, v);
                    else arrange48_rare(S, cls, info, p, r, s, v);
                    const int rr = (int)(e.w & 0xFFu), jj = (int)((e.w >> 8) & 0xFFu);
                    tc48_store_a(T, rr, jj, v);
                    const float g = __half2float(__ushort_as_half((unsigned short)(e.w >> 16)));
                    T.gain[jj][rr] = gain_mode == 0 ? g : g * S.invnorm[info_m(info)];
                }
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // generic writes -> MMA reads
        tc_fence_before();
        __syncthreads();
        if (T.status) break;                                   // uniform: set only before the barrier
        // ---- 4. one thread issues 2 x 6 MMA steps and commits them to the barrier
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; half++) {
                const uint32_t a0 = smem_u32(T.A[half]), b0 = smem_u32(T.B[half]);
#pragma unroll
                for (int s = 0; s < kTcK / 16; s++) {
                    const uint64_t ad = umma_desc(a0 + 2 * s * kTcALbo, kTcALbo, kTcSbo);
                    const uint64_t bd = umma_desc(b0 + 2 * s * kTcBLbo, kTcBLbo, kTcSbo);
                    asm volatile(
                        "{\n\t.reg .pred p;\n\t"
                        "setp.ne.b32 p, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                        ::"r"(tmem + (uint32_t)(half * kTcN)), "l"(ad), "l"(bd), "r"(kTcIdesc), "r"((uint32_t)s));
                }
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                         ::"r"(smem_u32(&T.mbar_mma)) : "memory");
        }
        pending = true;
        pphase = phase;
    }
    // ---- the last round's products (T.status is uniform here: nothing wrote it since the
    // last barrier)
    if (c0 < c1 && !T.status) {
        const float gep = T.gain[eslot][em];
        if (tc48_wait_mma(T, phase, mma_tries)) {
            pending = false;
            tc_fence_after();
            tc48_epilogue(etaddr, gep, yacc);
        } else if (lane == 0) {
            atomicOr(&T.status, 1u);
        }
    }
    // ---- sum the 8 slots of each row (in the A tiles, free now) and add the row sums into y
    __syncthreads();
    float *yred = reinterpret_cast<float *>(T.A[0]);             // [kTcRows][16]
    for (int i = tid; i < kTcRows * 16; i += kTc48Threads) yred[i] = 0.f;
    __syncthreads();
    if (!T.status) {
#pragma unroll
        for (int b = 0; b < 16; b++) atomicAdd(&yred[em * 16 + b], yacc[b]);
    }
    __syncthreads();
    for (int i = tid; i < kTcRows * 16; i += kTc48Threads) {
        const int m = i >> 4, b = i & 15;
        if (b < batch && row0 + m < rows && c0 < c1 && !T.status) atomicAdd(Y + (long long)b * rows + row0 + m, yred[i]);
    }
    if (tid == 0 && T.status) atomicOr(flags, kFlagWaitTimeout);
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicOr(flags, kFlagIndexRange);
    // ---- free the accumulator columns.  After a wait gave up, the committed MMAs may still be
    // writing them: every thread waits again (at most kMmaWaitTries polls) for the last commit,
    // and the columns are released only if it arrived; otherwise they are left allocated (the
    // flag is raised) rather than freed under the running MMAs.
    if (__syncthreads_or(pending)) {
        bool done = false;
        for (uint32_t it = 0; it < kMmaWaitTries && !done; it++) done = mbar_try_wait_parity(smem_u32(&T.mbar_mma), pphase);
        if (!__syncthreads_and(done)) return;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTc48TmemCols));
}

}  // namespace llvq
