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
