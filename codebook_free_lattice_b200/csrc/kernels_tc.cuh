// kernels_tc.cuh -- tile shapes, descriptors and fences of the small-batch product on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in TMEM), sm_100a only; the kernel is
// k_gemm_tc48 (kernels_tc48.cuh).
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
// step LBO apart (A: 2048 B, B: 1024 B).
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

// instruction descriptor: D f32, A and B f16, both K-major, N = 64, M = 128
constexpr uint32_t kTcIdesc = (1u << 4) | ((uint32_t)(kTcN >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);

// shared-memory matrix descriptor, K-major, no swizzle (descriptor version 1)
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

}  // namespace llvq
