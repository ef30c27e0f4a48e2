// device_common.cuh -- bit-level helpers shared by the LLVQ decoders (sm_100a).
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace llvq {

constexpr int kPdepEntries = 6561;   // sum over 8-bit masks m of 2^popcount(m)

// Cooperative copy of a read-only table image into shared memory (16-byte units).
__device__ __forceinline__ void load_smem_image(void *dst, const void *src, size_t bytes) {
    const int4 *s = reinterpret_cast<const int4 *>(src);
    int4 *d = reinterpret_cast<int4 *>(dst);
    const size_t n = bytes / 16;
    for (size_t i = threadIdx.x; i < n; i += blockDim.x) d[i] = __ldg(s + i);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ bool mbar_try_wait_parity(uint32_t bar, uint32_t parity) {
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

// Table images into shared memory with the bulk-copy engine: one bulk copy per region (sizes
// multiples of 16 bytes, both addresses 16-byte aligned) tracked by the mbarrier `bar`, then a
// bounded wait; a false return (in every thread) means a wait gave up, and the caller skips its
// work, raises a flag and returns.
constexpr uint32_t kBulkWaitTries = 1u << 22;
// The first half: thread 0 initialises the mbarrier, announces the bytes and starts the copies;
// ends with a CTA barrier (the mbarrier is initialised before anyone polls it).
template <int N>
__device__ __forceinline__ void bulk_load_issue(void *const (&dst)[N], const void *const (&src)[N],
                                                const uint32_t (&bytes)[N], unsigned long long *bar) {
    const uint32_t b = smem_u32(bar);
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        uint32_t total = 0;
#pragma unroll
        for (int i = 0; i < N; i++) total += bytes[i];
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(b), "r"(total) : "memory");
#pragma unroll
        for (int i = 0; i < N; i++)
            asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                         ::"r"(smem_u32(dst[i])), "l"(src[i]), "r"(bytes[i]), "r"(b) : "memory");
    }
    __syncthreads();
}
// The second half: every thread waits for the bytes, for at most first_tries polls; false in every
// thread if any wait gave up, after a second wait (at most kBulkWaitTries polls) so that no copy is
// still writing the shared memory the CTA is about to release.  Ends with a CTA barrier.
__device__ __forceinline__ bool bulk_load_wait(unsigned long long *bar, uint32_t first_tries) {
    const uint32_t b = smem_u32(bar);
    bool done = false;
    for (uint32_t it = 0; it < first_tries && !done; it++) done = mbar_try_wait_parity(b, 0);
    if (__syncthreads_and(done) != 0) return true;
    for (uint32_t it = 0; it < kBulkWaitTries && !done; it++) done = mbar_try_wait_parity(b, 0);
    __syncthreads();
    return false;
}
// Both halves.
template <int N>
__device__ __forceinline__ bool bulk_load_smem(void *const (&dst)[N], const void *const (&src)[N],
                                               const uint32_t (&bytes)[N], unsigned long long *bar,
                                               uint32_t first_tries = kBulkWaitTries) {
    bulk_load_issue(dst, src, bytes, bar);
    return bulk_load_wait(bar, first_tries);
}

// int8 x4 -> two half2 (exact): (b ^ 0x80) + 1024 is the fp16 with bits 0x64XX; minus 1152 = b
__device__ __forceinline__ void i8x4_to_h2x2(uint32_t w, uint32_t &lo, uint32_t &hi) {
    const uint32_t u = w ^ 0x80808080u;
    const uint32_t l = __byte_perm(u, 0x64646464u, 0x4140);     // coordinates 0, 1
    const uint32_t h = __byte_perm(u, 0x64646464u, 0x4342);     // coordinates 2, 3
    const __half2 bias = __halves2half2(__ushort_as_half((unsigned short)0x6480),
                                        __ushort_as_half((unsigned short)0x6480));
    const __half2 a = __hsub2(*reinterpret_cast<const __half2 *>(&l), bias);
    const __half2 b = __hsub2(*reinterpret_cast<const __half2 *>(&h), bias);
    lo = *reinterpret_cast<const uint32_t *>(&a);
    hi = *reinterpret_cast<const uint32_t *>(&b);
}

// acc + w.lo * x.lo + w.hi * x.hi for fp16 pairs w, x with fp32 accumulation: each product of two
// fp16 values is exact in fp32 and is added with one rounding (mixed-precision FMA, sm_100).
__device__ __forceinline__ float fma2_f16_f32(uint32_t w, uint32_t x, float acc) {
    asm("{\n\t.reg .f16 w0, w1, x0, x1;\n\t"
        "mov.b32 {w0, w1}, %1;\n\t"
        "mov.b32 {x0, x1}, %2;\n\t"
        "fma.rn.f32.f16 %0, w0, x0, %0;\n\t"
        "fma.rn.f32.f16 %0, w1, x1, %0;\n\t}"
        : "+f"(acc)
        : "r"(w), "r"(x));
    return acc;
}

// bit k of a nibble -> byte k (0x01)
__device__ __forceinline__ uint32_t nibble_to_bytes(uint32_t nib) {
    return (nib * 0x00204081u) & 0x01010101u;
}
// bit 0 of byte k -> bit k of a nibble
__device__ __forceinline__ uint32_t bytes_to_nibble(uint32_t b) {
    return ((b & 0x01010101u) * 0x01020408u) >> 24 & 0xFu;
}

// Exact double of a small non-negative integer (n < 2^31) built from its bits (2^52 + n) and
// one subtraction, keeping the work off the conversion pipe.
__device__ __forceinline__ double small_to_double(uint32_t n) {
    return __hiloint2double(0x43300000, (int)n) - 0x1p52;
}

// Deposit the low bits of src on the set bits of a 24-bit mask, lowest bit first, through a
// byte-wise table: tab[off[m] + b] = bits b spread over the set bits of the byte mask m.
__device__ __forceinline__ uint32_t pdep24(uint32_t src, uint32_t mask, const uint16_t *off,
                                           const uint8_t *tab) {
    uint32_t out = 0;
#pragma unroll
    for (int j = 0; j < 3; j++) {
        const uint32_t mb = (mask >> (8 * j)) & 0xFFu;
        const uint32_t n = __popc(mb);
        out |= (uint32_t)tab[off[mb] + (src & ((1u << n) - 1u))] << (8 * j);
        src >>= n;
    }
    return out;
}

// Signs and final bytes.  F has one bit per coordinate: odd coset -> |x_i| = 1 (mod 4),
// even coset -> x_i != 0.  odd: x_i = 1 (mod 4) exactly on the codeword T, so the negative
// coordinates are T xor F.  even: bit j of s negates the j-th nonzero coordinate (ascending),
// skipping the highest coordinate of the codeword S, whose sign makes the number of negative
// coordinates on S congruent to sum|x|/4 (parity) mod 2.  mag[q] holds |x| for coordinates
// 4q..4q+3; the result v[q] holds the signed int8 coordinates.
__device__ __forceinline__ void apply_signs(bool odd, uint32_t word, uint32_t s, uint32_t F,
                                            uint32_t parity, const uint32_t mag[6], bool ok,
                                            const uint16_t *pdep_off, const uint8_t *pdep,
                                            uint32_t v[6]) {
    uint32_t neg;
    if (odd) {
        neg = word ^ F;
    } else {
        const uint32_t topbit = word ? (0x80000000u >> __clz(word)) : 0u;
        neg = pdep24(s, F & ~topbit, pdep_off, pdep);
        neg |= ((__popc(neg & word) ^ parity) & 1u) ? topbit : 0u;
    }
#pragma unroll
    for (int q = 0; q < 6; q++) {
        const uint32_t nb = nibble_to_bytes((neg >> (4 * q)) & 0xFu);
        v[q] = ok ? (mag[q] ^ (nb * 0xFFu)) + nb : 0u;
    }
}

}  // namespace llvq
