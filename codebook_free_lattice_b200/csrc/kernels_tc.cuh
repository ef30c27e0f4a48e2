// kernels_tc.cuh -- small-batch fused decode-and-multiply on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in TMEM), sm_100a only.
//
// "Leech Lattice Vector Quantization for Efficient LLM Compression", papernotes.org notes,
// 方法详解 / 关键设计 4: blocks are decoded on chip and multiplied with the activations without
// writing dequantized weights to global memory.  Here the decoded blocks of a 128-row tile go to
// shared memory as exact fp16 integers, and one MMA per 16-wide K step multiplies them with a
// block-diagonal activation tile:
//
//   A [128 rows][96 k]  : the 4 blocks (4 x 24 k) of a K chunk, fp16 integers (exact)
//   B [64 n][96 k]      : n = 16 * jj + b holds x_b on block jj's 24 columns, zero elsewhere
//   D [128][64] (TMEM)  : D[m][16 jj + b] = <v(m, jj), x_b(jj)>, the per-block partial dots
//
// so the per-block gains apply afterwards in fp32 (y_b[m] += g(m, jj) * D[m][16 jj + b]) and
// no gain is rounded to fp16.  Operands use the no-swizzle K-major layout: 8-row x 16-byte core
// matrices, rows 16 B apart, 8-row groups SBO = 128 B apart, the two 8-element K halves of a
// step LBO apart (A: 2048 B, B: 1024 B).  One CTA = one 128-row tile x a range of K chunks;
// several CTAs per tile (split K) add into the zeroed output with atomics.
#pragma once
#include "kernels.cuh"

namespace llvq {


constexpr int kTcRows = 128;                  // UMMA M
constexpr int kTcBlocks = 4;                  // 24-weight blocks per K chunk
constexpr int kTcK = kTcBlocks * 24;          // 96 = 6 MMA steps of 16
constexpr int kTcN = kTcBlocks * 16;          // 64 = 4 blocks x 16 batch slots
constexpr int kTcASize = kTcK / 8 * kTcRows * 16;   // 24576 B
constexpr int kTcBSize = kTcK / 8 * kTcN * 16;      // 12288 B
constexpr uint32_t kTcALbo = kTcRows * 16;          // 2048 B between K halves
constexpr uint32_t kTcBLbo = kTcN * 16;             // 1024 B between K halves
constexpr uint32_t kTcSbo = 128;                    // 8 rows x 16 B
constexpr uint32_t kTcTmemCols = 64;                // fp32 accumulator columns (power of 2, >= 32)

// instruction descriptor: D f32, A and B f16, both K-major, N = 64, M = 128
constexpr uint32_t kTcIdesc = (1u << 4) | ((uint32_t)(kTcN >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// shared-memory matrix descriptor, K-major, no swizzle (descriptor version 1)
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}


template <class D>
struct TcSmem {
    typename D::Smem tables;
    __align__(128) unsigned char A[kTcASize];          // reused for the final row sums
    __align__(128) unsigned char B[kTcBSize];
    float gain[kTcBlocks][kTcRows];
    unsigned long long mbar;
    uint32_t tmem_base;
    uint32_t status;
};
static_assert(kTcRows * 16 * sizeof(float) <= kTcASize, "row sums must fit in the A tile");

template <class D>
constexpr int tc_ctas_per_sm() { return D::kWordBytes == 8 ? 2 : 1; }

// grid = (row tiles, K splits); 512 threads: decode maps thread t to (row t / 4, block t % 4) so
// each group of four threads reads one row's 32 consecutive word bytes; the epilogue maps warp w
// to TMEM lanes 32 (w % 4).. (rows) and block w / 4 (16 accumulator columns).
template <class D>
__global__ void __launch_bounds__(512, tc_ctas_per_sm<D>()) k_gemm_tc(typename D::Args args, const typename D::Word *__restrict__ words,
                                                   long long pitch, int rows, int nb, int batch, int gain_mode,
                                                   const __half *__restrict__ gains, const __half *__restrict__ X,
                                                   float *__restrict__ Y, int chunks_per_split,
                                                   unsigned *__restrict__ flags) {
    extern __shared__ __align__(128) unsigned char smem_tc[];
    TcSmem<D> &S = *reinterpret_cast<TcSmem<D> *>(smem_tc);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    load_smem_image(&S.tables, args.image, sizeof(typename D::Smem));
    for (int i = tid; i < kTcBSize / 16; i += blockDim.x) reinterpret_cast<uint4 *>(S.B)[i] = make_uint4(0, 0, 0, 0);
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&S.mbar)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        S.status = 0;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr(&S.tmem_base)), "r"(kTcTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    const int row0 = blockIdx.x * kTcRows;
    const int nchunks = (nb + kTcBlocks - 1) / kTcBlocks;
    const int c0 = blockIdx.y * chunks_per_split;
    const int c1 = min(c0 + chunks_per_split, nchunks);
    const long long K = (long long)nb * 24;
    const int dr = tid >> 2, djj = tid & 3;                // decode role
    const int lg = warp & 3, ejj = warp >> 2;              // epilogue role
    const int em = lg * 32 + lane;
    float yacc[16];
#pragma unroll
    for (int b = 0; b < 16; b++) yacc[b] = 0.f;
    bool bad = false;
    uint32_t phase = 0;

    for (int ch = c0; ch < c1; ch++) {
        const int j0 = ch * kTcBlocks;
        // ---- decode one block per thread into A (fp16 integers) and its gain into S.gain
        {
            const int r = row0 + dr, j = j0 + djj;
            uint32_t h[12] = {0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0};
            float scale = 0.f;
            if (r < rows && j < nb) {
                const typename D::Word w = D::load(words + (long long)r * pitch + j);
                uint32_t v[6];
                int m;
                bad |= !D::decode(w, S.tables, args, v, m);
#pragma unroll
                for (int q = 0; q < 6; q++) i8x4_to_h2x2(v[q], h[2 * q], h[2 * q + 1]);
                if (gain_mode == 0) scale = __half2float(__ldg(gains + (long long)r * nb + j));
                else scale = __half2float(__ldg(gains + (long long)r * 256 + D::gain_code(w))) * D::invnorm(S.tables, m);
            }
#pragma unroll
            for (int q = 0; q < 3; q++)
                *reinterpret_cast<uint4 *>(S.A + (3 * djj + q) * kTcALbo + dr * 16) =
                    make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
            S.gain[djj][dr] = scale;
        }
        // ---- B: block-diagonal activations, 3 x 16 B per (block, batch slot)
        if (tid < kTcBlocks * 16 * 3) {
            const int q = tid % 3, nidx = tid / 3;             // n = 16 jj + b
            const int jj = nidx >> 4, b = nidx & 15;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (b < batch && j0 + jj < nb)
                val = __ldg(reinterpret_cast<const uint4 *>(X + b * K + (long long)(j0 + jj) * 24 + 8 * q));
            *reinterpret_cast<uint4 *>(S.B + (3 * jj + q) * kTcBLbo + nidx * 16) = val;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // generic writes -> MMA reads
        tc_fence_before();
        __syncthreads();
        // ---- one thread issues the 6 MMA steps and commits them to the barrier
        if (tid == 0) {
            tc_fence_after();
            const uint32_t a0 = smem_addr(S.A), b0 = smem_addr(S.B);
#pragma unroll
            for (int s = 0; s < kTcK / 16; s++) {
                const uint64_t ad = umma_desc(a0 + 2 * s * kTcALbo, kTcALbo, kTcSbo);
                const uint64_t bd = umma_desc(b0 + 2 * s * kTcBLbo, kTcBLbo, kTcSbo);
                asm volatile(
                    "{\n\t.reg .pred p;\n\t"
                    "setp.ne.b32 p, %4, 0;\n\t"
                    "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                    ::"r"(tmem), "l"(ad), "l"(bd), "r"(kTcIdesc), "r"((uint32_t)s));
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                         ::"r"(smem_addr(&S.mbar)) : "memory");
        }
        // ---- bounded wait for the MMAs, then read this warp's 32 rows x 16 columns
        {
            bool done = false;
            for (int it = 0; it < (1 << 20) && !done; it++) done = mbar_try_wait(smem_addr(&S.mbar), phase);
            if (!done) atomicOr(&S.status, 1u);
        }
        phase ^= 1u;
        __syncthreads();
        if (S.status) break;                                   // uniform: read after the barrier
        tc_fence_after();
        uint32_t d[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
            : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]), "=r"(d[6]), "=r"(d[7]),
              "=r"(d[8]), "=r"(d[9]), "=r"(d[10]), "=r"(d[11]), "=r"(d[12]), "=r"(d[13]), "=r"(d[14]), "=r"(d[15])
            : "r"(tmem + ((uint32_t)(lg * 32) << 16) + (uint32_t)(ejj * 16)));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        const float g = S.gain[ejj][em];
#pragma unroll
        for (int b = 0; b < 16; b++) yacc[b] = fmaf(g, __uint_as_float(d[b]), yacc[b]);
        tc_fence_before();
        __syncthreads();                                       // A, B and TMEM free for the next chunk
    }
    // ---- sum the four block columns of each row (in the A tile, free now) and add the row sums
    //      into the output, which the launch zeroed (several K splits add into each row)
    __syncthreads();
    float *yred = reinterpret_cast<float *>(S.A);                 // [kTcRows][16]
    for (int i = tid; i < kTcRows * 16; i += blockDim.x) yred[i] = 0.f;
    __syncthreads();
    if (!S.status) {
#pragma unroll
        for (int b = 0; b < 16; b++) atomicAdd(&yred[em * 16 + b], yacc[b]);
    }
    __syncthreads();
    for (int i = tid; i < kTcRows * 16; i += blockDim.x) {
        const int m = i >> 4, b = i & 15;
        if (b < batch && row0 + m < rows && c0 < c1 && !S.status) atomicAdd(Y + (long long)b * rows + row0 + m, yred[i]);
    }
    if (tid == 0 && S.status) atomicOr(flags, kFlagWaitTimeout);
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicOr(flags, 0x1u);
    // ---- free the accumulator columns (all TMEM reads have completed above)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols));
}

}  // namespace llvq
