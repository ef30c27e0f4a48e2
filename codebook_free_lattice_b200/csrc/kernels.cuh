// kernels.cuh -- decode and fused decode-and-multiply kernels generic over the index budget's
// decoder (Dec48 for the allocation-free decode; Dec72, Dec96 for every product and decode at 3
// and 4 bits), and the encoder kernels.  "Leech Lattice Vector Quantization for Efficient LLM
// Compression", papernotes.org notes, 方法详解 / 关键设计 4: each block is decoded to its 24-dim
// integer vector in registers and multiplied with the activations; dequantized weights never
// reach global memory.
#pragma once
#include "codec48.cuh"
#include "codec72.cuh"
#include "encode48.cuh"
#include "encode72.cuh"
#include "encode96.cuh"

namespace llvq {

constexpr unsigned kFlagIndexRange = 0x1u;   // an index >= N_M was met (LLVQ_FLAG_INDEX_RANGE)
constexpr unsigned kFlagWaitTimeout = 0x2u;  // a bounded wait gave up (LLVQ_FLAG_WAIT_TIMEOUT)
constexpr unsigned kFlagNotCoded = 0x4u;     // an encoded vector is not a coded point (LLVQ_FLAG_NOT_CODED)
constexpr unsigned kFlagSearchInput = 0x8u;  // a searched row held a NaN or an infinity (LLVQ_FLAG_SEARCH_INPUT)

// Decode n packed words into int8 [n][24].
template <class D>
__global__ void __launch_bounds__(512, D::kCtasPerSm) k_decode(typename D::Args args,
                                                  const typename D::Word *__restrict__ words,
                                                  long long n, int8_t *__restrict__ out,
                                                  unsigned *__restrict__ flags) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    typename D::Smem &S = *reinterpret_cast<typename D::Smem *>(smem_raw);
    load_smem_image(&S, args.image, sizeof(typename D::Smem));
    __syncthreads();
    bool bad = false;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n;
         t += (long long)gridDim.x * blockDim.x) {
        uint32_t v[6];
        int m;
        bad |= !D::decode(D::load(words + t), S, args, v, m);
        uint2 *o = reinterpret_cast<uint2 *>(out + t * 24);
        o[0] = make_uint2(v[0], v[1]);
        o[1] = make_uint2(v[2], v[3]);
        o[2] = make_uint2(v[4], v[5]);
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicOr(flags, kFlagIndexRange);
}

// Encode n lattice points (int8 [n][24]) into 48-bit packed words (gain code 0).
__global__ void __launch_bounds__(512, 2) k_encode48(const EncSmem48 *__restrict__ image, unsigned long long npoints,
                                                     const int8_t *__restrict__ vecs, long long n,
                                                     unsigned long long *__restrict__ words,
                                                     unsigned *__restrict__ flags) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    EncSmem48 &E = *reinterpret_cast<EncSmem48 *>(smem_raw);
    load_smem_image(&E, image, sizeof(EncSmem48));
    __syncthreads();
    bool bad = false;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n;
         t += (long long)gridDim.x * blockDim.x) {
        const uint2 *src = reinterpret_cast<const uint2 *>(vecs + t * 24);
        const uint2 a = __ldg(src), b = __ldg(src + 1), c = __ldg(src + 2);
        const uint32_t xw[6] = {a.x, a.y, b.x, b.y, c.x, c.y};
        unsigned long long I;
        bad |= !encode48(xw, E, npoints, I);
        words[t] = I;
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicOr(flags, kFlagNotCoded);
}

// Encode n lattice points (int8 [n][24]) into 72-bit packed words (16 bytes, gain code 0).
__global__ void __launch_bounds__(512, 2) k_encode72(const EncSmem72 *__restrict__ image,
                                                     const Rec72 *__restrict__ recs,
                                                     const unsigned long long *__restrict__ keys,
                                                     unsigned long long np_lo, unsigned long long np_hi,
                                                     const int8_t *__restrict__ vecs, long long n,
                                                     ulonglong2 *__restrict__ words, unsigned *__restrict__ flags) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    EncSmem72 &E = *reinterpret_cast<EncSmem72 *>(smem_raw);
    load_smem_image(&E, image, sizeof(EncSmem72));
    __syncthreads();
    bool bad = false;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n;
         t += (long long)gridDim.x * blockDim.x) {
        const uint2 *src = reinterpret_cast<const uint2 *>(vecs + t * 24);
        const uint2 a = __ldg(src), b = __ldg(src + 1), c = __ldg(src + 2);
        const uint32_t xw[6] = {a.x, a.y, b.x, b.y, c.x, c.y};
        unsigned long long lo, hi;
        bad |= !encode72(xw, E, recs, keys, np_lo, np_hi, lo, hi);
        words[t] = make_ulonglong2(lo, hi);
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicOr(flags, kFlagNotCoded);
}

// The 96-bit class keys: the unary code of the class's magnitude counts from the coset's
// largest magnitude down, from the class records (one thread per class).
__global__ void k_keys96(const Rec96 *__restrict__ recs, long long ncls, unsigned long long *__restrict__ keys) {
    const long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= ncls) return;
    const ulonglong2 *rp = reinterpret_cast<const ulonglong2 *>(recs + c);
    const uint32_t meta = (uint32_t)(__ldg(rp).y >> 32);
    const uint4 cumv = __ldg(reinterpret_cast<const uint4 *>(rp + 2));
    const uint4 valv = __ldg(reinterpret_cast<const uint4 *>(rp + 3));
    const bool odd = meta & kMeta96Odd;
    const uint32_t cw[4] = {cumv.x, cumv.y, cumv.z, cumv.w}, vw[4] = {valv.x, valv.y, valv.z, valv.w};
    unsigned long long key = 0;
    for (int b = 29; b >= 0; b--) {
        if (odd && b == 29) continue;
        const uint32_t v = 2u * (uint32_t)b + (odd ? 1u : 0u);
        uint32_t cnt = 0, prev = 0;
        for (int g = 0; g < 16; g++) {
            const uint32_t cg = ((cw[g >> 2] >> (8 * (g & 3))) & 0xFFu) - 0x7Fu;
            const uint32_t vg = (vw[g >> 2] >> (8 * (g & 3))) & 0xFFu;
            if (cg > prev && vg == v) cnt = cg - prev;
            prev = cg;
        }
        key = (key << (cnt + 1u)) | (((1ull << cnt) - 1ull) << 1);
    }
    keys[c] = key;
}

// Encode n lattice points (int8 [n][24]) into 96-bit packed words (16 bytes, gain code 0).
__global__ void __launch_bounds__(256, 2) k_encode96(const EncSmem96 *__restrict__ image,
                                                     const Rec96 *__restrict__ recs,
                                                     const unsigned long long *__restrict__ keys,
                                                     unsigned long long np_lo, unsigned long long np_hi,
                                                     const int8_t *__restrict__ vecs, long long n,
                                                     ulonglong2 *__restrict__ words, unsigned *__restrict__ flags) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    EncSmem96 &E = *reinterpret_cast<EncSmem96 *>(smem_raw);
    load_smem_image(&E, image, sizeof(EncSmem96));
    __syncthreads();
    bool bad = false;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n;
         t += (long long)gridDim.x * blockDim.x) {
        const uint2 *src = reinterpret_cast<const uint2 *>(vecs + t * 24);
        const uint2 a = __ldg(src), b = __ldg(src + 1), c = __ldg(src + 2);
        const uint32_t xw[6] = {a.x, a.y, b.x, b.y, c.x, c.y};
        unsigned long long lo, hi;
        bad |= !encode96(xw, E, recs, keys, np_lo, np_hi, lo, hi);
        words[t] = make_ulonglong2(lo, hi);
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicOr(flags, kFlagNotCoded);
}

template <class D, int BATCH>
constexpr int gemm_ctas_per_sm() { return BATCH == 1 ? D::kCtasPerSm : 2; }

// Shared accumulator slots per (batch row, output row): one per lane up to batch 7; from batch 8
// up, lanes l, l + 8, l + 16, l + 24 share a slot, which keeps the accumulators of a 97-row tile
// at batch 16 within 50 KB (two CTAs per SM).
template <int BATCH>
constexpr int gemm_acc_slots() { return BATCH <= 7 ? 32 : 8; }

// Fused decode and multiply, batch `batch` <= BATCH (BATCH 1..7 exact, 8 or 16 with a runtime
// batch).  Each CTA owns a contiguous range of rows;
// its threads walk the range's blocks in row-major order (each warp reads 32 consecutive
// packed words), decode each block once and form scale * <v, x_b> for every batch row.
// Contributions go to shared-memory accumulators acc[b][row][slot] by atomic add (slot = lane up
// to batch 7: only warps of the same CTA meet on a word); at the end one warp per (b, row) sums
// the slots and writes the output.
// gain: direct mode -> fp16 gains[row][nb]; table mode -> fp16 gains[row][256] indexed by the
// word's 8-bit code, times 1/|v| = 1/(4 sqrt(m)) (shape-gain: unit direction times gain).
template <class D, int BATCH>
__global__ void __launch_bounds__(512, gemm_ctas_per_sm<D, BATCH>()) k_gemm(
    typename D::Args args, const typename D::Word *__restrict__ words, long long pitch, int rows, int nb,
    uint32_t nb_recip, int gain_mode, const __half *__restrict__ gains, const __half *__restrict__ X,
    float *__restrict__ Y, int rows_per_cta, int batch, unsigned *__restrict__ flags) {
    constexpr int SLOTS = gemm_acc_slots<BATCH>();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    typename D::Smem &S = *reinterpret_cast<typename D::Smem *>(smem_raw);
    float *acc = reinterpret_cast<float *>(smem_raw + sizeof(typename D::Smem));  // [BATCH][rpc][SLOTS]
    load_smem_image(&S, args.image, sizeof(typename D::Smem));
    for (int i = threadIdx.x; i < BATCH * rows_per_cta * SLOTS; i += blockDim.x) acc[i] = 0.f;
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
            const typename D::Word w = D::load(words + (long long)r * pitch + j);
            uint32_t v[6];
            int m;
            bad |= !D::decode(w, S, args, v, m);
            float scale;
            if (gain_mode == 0) {
                scale = __half2float(__ldg(gains + (long long)r * nb + j));
            } else {
                scale = __half2float(__ldg(gains + (long long)r * 256 + D::gain_code(w))) * D::invnorm(S, m);
            }
            float wv[24];
#pragma unroll
            for (int q = 0; q < 6; q++)
#pragma unroll
                for (int e = 0; e < 4; e++) wv[4 * q + e] = (float)(int8_t)(v[q] >> (8 * e));
#pragma unroll
            for (int bb = 0; bb < BATCH; bb++) {
                if (BATCH >= 8 && bb >= batch) break;
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
                atomicAdd(&acc[(bb * rows_per_cta + rl) * SLOTS + (lane & (SLOTS - 1))], scale * dot);
            }
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    const int nbatch = BATCH >= 8 ? batch : BATCH;
    for (int i = warp; i < nbatch * nrows; i += blockDim.x >> 5) {
        const int bb = i / nrows, rl = i - bb * nrows;
        float sum = lane < SLOTS ? acc[(bb * rows_per_cta + rl) * SLOTS + lane] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        if (lane == 0) Y[(long long)bb * rows + row0 + rl] = sum;
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicOr(flags, kFlagIndexRange);
}

}  // namespace llvq
