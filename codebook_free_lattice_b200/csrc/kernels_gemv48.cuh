// kernels_gemv48.cuh -- 48-bit fused decode-and-multiply for batches 1..7 (the 2-bit GEMV).
//
// "Leech Lattice Vector Quantization for Efficient LLM Compression", papernotes.org notes,
// 方法详解 / 关键设计 2 and 4: each block's packed index is decoded to its 24-dim integer vector in
// registers and multiplied with the activations; dequantized weights never reach global memory.
//
// One 1024-thread CTA per SM owns a row range.  Its warps take slices of 32 consecutive blocks
// from a shared counter, classify them (one block per lane) and append each block's digits to one
// of two private record rings, odd coset or even coset.  Whenever a ring holds 32 records the warp
// decodes them together, so all lanes of a warp run the same decode.  Blocks of the rare classes
// (odd with five magnitude groups, even off the table path) are decoded where they are met.  Each
// block's product is added to y in global memory by a reduction (no return value), so no warp
// waits for another: the CTA zeroes its rows of y before its warps start, and a warp that runs out
// of slices decodes what is left in its rings and exits.  An even-coset block's complement code
// sequence (a global table) is requested when the block is classified and its record is written
// to the ring one slice later, so the load overlaps the warp's other work.  The table image is
// copied to shared memory before the kernel waits for the kernels it depends on (programmatic
// dependent launch), so that copy overlaps the end of the previous kernel on the stream; the
// activations are staged in shared memory when they fit.
#pragma once
#include "kernels_bin48.cuh"

namespace llvq {

constexpr int kGvThreads = 1024;
constexpr int kGvWarps = kGvThreads / 32;
constexpr int kGvRing = 64;                   // records per ring (a warp drains a ring at 32)

// table image, the rings [warp][odd, even][kGvRing], the slice counter and the table mbarrier,
// then (when staged) the activations [batch][nb * 24] fp16
__host__ __device__ constexpr size_t gv48_fixed_smem() {
    return sizeof(SmemGv48) + sizeof(BinRec) * (kGvWarps * 2 * kGvRing) + 16;
}
__host__ __device__ constexpr size_t gv48_smem_bytes(int batch, int nb, bool stage_x) {
    return gv48_fixed_smem() + (stage_x ? (size_t)batch * nb * 48 : 0);
}

struct GvArgs {
    const SmemGv48 *image;
    unsigned long long npoints;
    const uint32_t *tabC;                     // complement arrangement table (even table path)
    const unsigned long long *words;
    long long pitch;
    int rows, nb;
    uint32_t nb_recip;                        // ceil(2^32 / nb): block index -> row by a multiply-high
    int gain_mode;
    const __half *gains, *X;
    float *Y;
    int rows_per_cta;
    uint32_t wait_tries;                      // polls of the table copy's first wait
};

// The decoded block (12 fp16 pairs, exact small integers) times the activations, scaled; the
// activations from shared memory (XS) or global memory.
template <int BATCH, bool XS>
__device__ __forceinline__ void gv_dot(const uint32_t wh[12], float scale, const __half *__restrict__ X,
                                       const __half *xs, long long K, int j, float d[BATCH]) {
#pragma unroll
    for (int bb = 0; bb < BATCH; bb++) {
        const uint4 *xp = reinterpret_cast<const uint4 *>((XS ? xs : X) + bb * K + (long long)j * 24);
        float d0 = 0.f, d1 = 0.f;
#pragma unroll
        for (int c = 0; c < 3; c++) {
            const uint4 raw = XS ? xp[c] : __ldg(xp + c);
            d0 = fma2_f16_f32(wh[4 * c + 0], raw.x, d0);
            d1 = fma2_f16_f32(wh[4 * c + 1], raw.y, d1);
            d0 = fma2_f16_f32(wh[4 * c + 2], raw.z, d0);
            d1 = fma2_f16_f32(wh[4 * c + 3], raw.w, d1);
        }
        d[bb] = scale * (d0 + d1);
    }
}

// Steps 3-5 of one record of the given kind (0 odd fast path, 1 even table path, 2 rare): the
// block as 12 fp16 pairs.
template <int KIND>
__device__ __forceinline__ void gv_decode(const GvArgs &a, const SmemGv48 &S, const BinRec e, int cls, uint32_t r,
                                          uint32_t info, uint32_t wh[12]) {
    const unsigned long long p = (unsigned long long)((e.y >> 21) & 1u) << 32 | e.x;
    if constexpr (KIND == 0) {
        arrange_odd48_f16(S, cls, p, r, wh);
    } else if constexpr (KIND == 1) {
        // x: the complement's code sequence (fetched at classification), y bits 21..31: p_S
        arrange_even48_f16(S, cls, info, e.y >> 21, r, e.z & 0xFFFFFFu, e.x, wh);
    } else {
        const uint32_t word = (info & kInfoOdd) ? odd_codeword48(S, r)
                                                : S.gweight[min((S.c_info2[cls] & 0xFFFu) + r, 4095u)];
        uint32_t v[6];
        arrange48_word(S, cls, info, word, p, e.z & 0xFFFFFFu, true, v);
#pragma unroll
        for (int q = 0; q < 6; q++) i8x4_to_h2x2(v[q], wh[2 * q], wh[2 * q + 1]);
    }
}

// Decode a record and add its product to y (a reduction in global memory).  GAIN: 0 direct fp16
// gain per block, 1 per-row table indexed by the word's gain code.
template <int KIND, int BATCH, int GAIN, bool XS>
__device__ __forceinline__ void gv_consume(const GvArgs &a, const SmemGv48 &S, const __half *xs, const BinRec e,
                                           int row0) {
    const int cls = (int)(e.y & 0x1FFu);
    const uint32_t r = (e.y >> 9) & 0xFFFu;
    const uint32_t info = S.c_info[cls];
    const int rl = (int)(e.w & 0xFFFFu), j = (int)(e.w >> 16);
    const long long row = (long long)row0 + rl;
    const float scale = GAIN == 0 ? __half2float(__ldg(a.gains + row * a.nb + j))
                                  : __half2float(__ldg(a.gains + row * 256 + (e.z >> 24))) * S.invnorm[info_m(info)];
    uint32_t wh[12];
    gv_decode<KIND>(a, S, e, cls, r, info, wh);
    float d[BATCH];
    gv_dot<BATCH, XS>(wh, scale, a.X, xs, (long long)a.nb * 24, j, d);
#pragma unroll
    for (int bb = 0; bb < BATCH; bb++) atomicAdd(a.Y + (long long)bb * a.rows + row, d[bb]);
}

template <int BATCH, int GAIN, bool XS>
__global__ void __launch_bounds__(kGvThreads, 1) k_gemv48(GvArgs a, unsigned *__restrict__ flags) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SmemGv48 &S = *reinterpret_cast<SmemGv48 *>(smem_raw);
    BinRec *rings = reinterpret_cast<BinRec *>(smem_raw + sizeof(SmemGv48));
    int *slice_next = reinterpret_cast<int *>(rings + kGvWarps * 2 * kGvRing);
    unsigned long long *bar = reinterpret_cast<unsigned long long *>(slice_next + 2);
    __half *xs = reinterpret_cast<__half *>(bar + 1);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned lanes_below = (1u << lane) - 1u;
    const int rpc = a.rows_per_cta;
    const int row0 = blockIdx.x * rpc;
    const int nrows = max(0, min(rpc, a.rows - row0));
    const int nb = a.nb;
    const int total = nrows * nb;
    const int nslices = (total + 31) / 32;
    BinRec *ring_odd = rings + warp * 2 * kGvRing;
    BinRec *ring_even = ring_odd + kGvRing;

    // the next kernel on the stream may start its own table copy now; it waits (as this one does
    // below) for the kernels before it to finish before it touches their results
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (tid == 0) *slice_next = kGvWarps;      // slices 0..31 go to warps 0..31 directly
    {
        void *const dst[1] = {&S};
        const void *const src[1] = {a.image};
        const uint32_t bytes[1] = {(uint32_t)sizeof(SmemGv48)};
        bulk_load_issue(dst, src, bytes, bar);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int i = tid; i < BATCH * nrows; i += kGvThreads) {
        const int bb = i / nrows, rr = i - bb * nrows;
        a.Y[(long long)bb * a.rows + row0 + rr] = 0.f;
    }
    if constexpr (XS) {
        const int n16 = BATCH * nb * 3;                             // 16-byte units
        const uint4 *src = reinterpret_cast<const uint4 *>(a.X);
        uint4 *dst = reinterpret_cast<uint4 *>(xs);
        for (int i = tid; i < n16; i += kGvThreads) dst[i] = __ldg(src + i);
    }
    // the table copy's wait ends with a CTA barrier, which also orders the zeroed rows of y before
    // any reduction into them and the staged activations before their use
    if (!bulk_load_wait(bar, a.wait_tries)) {
        if (tid == 0) atomicOr(flags, kFlagWaitTimeout);
        return;
    }

    const bool dense = a.pitch == (long long)nb;
    const unsigned long long *wbase = a.words + (long long)row0 * a.pitch;
    auto word_at = [&](int t) -> unsigned long long {
        if (t >= total) return 0ull;
        if (dense) return __ldg(wbase + t);
        const int rl = nb == 1 ? t : (int)__umulhi((uint32_t)t, a.nb_recip);
        return __ldg(wbase + (long long)rl * a.pitch + (t - rl * nb));
    };

    bool bad = false;
    int oh = 0, ot = 0, eh = 0, et = 0;       // ring heads and tails (warp-uniform)
    // the previous slice's record, written to its ring one slice late (pk: 0 odd, 1 even, 3 none)
    BinRec prec;
    int pk = 3;
    prec.x = prec.y = prec.z = prec.w = 0u;
    auto append = [&](const BinRec &rec, int k) {
        const unsigned mo = __ballot_sync(0xFFFFFFFFu, k == 0);
        const unsigned me = __ballot_sync(0xFFFFFFFFu, k == 1);
        if (k == 0) ring_odd[(ot + __popc(mo & lanes_below)) & (kGvRing - 1)] = rec;
        if (k == 1) ring_even[(et + __popc(me & lanes_below)) & (kGvRing - 1)] = rec;
        ot += __popc(mo);
        et += __popc(me);
        __syncwarp();
        if (ot - oh >= 32) {
            gv_consume<0, BATCH, GAIN, XS>(a, S, xs, ring_odd[(oh + lane) & (kGvRing - 1)], row0);
            oh += 32;
        }
        if (et - eh >= 32) {
            gv_consume<1, BATCH, GAIN, XS>(a, S, xs, ring_even[(eh + lane) & (kGvRing - 1)], row0);
            eh += 32;
        }
        __syncwarp();
    };
    int sl = warp;                             // current slice (warp-uniform)
    unsigned long long w = sl < nslices ? word_at(sl * 32 + lane) : 0ull;
    while (sl < nslices) {
        int sn = 0;
        if (lane == 0) sn = atomicAdd(slice_next, 1);
        sn = __shfl_sync(0xFFFFFFFFu, sn, 0);
        const unsigned long long wn = sn < nslices ? word_at(sn * 32 + lane) : 0ull;
        const int t = sl * 32 + lane;
        // classify this slice; an even block on the table path requests its complement sequence
        const bool valid = t < total;
        const Cls48 cl = classify48(w, S, a.npoints);
        bad |= valid && !cl.ok;
        const bool enq = valid && cl.ok;
        const bool odd = cl.info & kInfoOdd;
        int kind = odd ? (info_val4(cl.info) == 0u ? 0 : 2) : ((cl.info & kInfoTable) ? 1 : 2);
        if (!enq) kind = 3;
        const int rl = valid ? (nb == 1 ? t : (int)__umulhi((uint32_t)t, a.nb_recip)) : 0;
        BinRec rec;
        rec.x = (uint32_t)cl.p;
        rec.y = (uint32_t)cl.cls | cl.r << 9 | (uint32_t)(cl.p >> 32) << 21;
        rec.z = cl.s | (uint32_t)((w >> 48) & 0xFFu) << 24;
        rec.w = (uint32_t)rl | (uint32_t)(t - rl * nb) << 16;
        if (kind == 1) {
            uint32_t pS;
            const uint32_t pC = even48_pC(S, cl.cls, (uint32_t)cl.p, pS);
            rec.x = __ldg(a.tabC + (S.c_offs[cl.cls] & 0x7FFFFu) + pC);
            rec.y = (uint32_t)cl.cls | cl.r << 9 | pS << 21;
        }
        if (kind == 2) gv_consume<2, BATCH, GAIN, XS>(a, S, xs, rec, row0);
        // the previous slice's records into the rings, full batches decoded
        append(prec, pk);
        prec = rec;
        pk = kind;
        w = wn;
        sl = sn;
    }
    append(prec, pk);
    // what is left in the rings
    if (lane < ot - oh) gv_consume<0, BATCH, GAIN, XS>(a, S, xs, ring_odd[(oh + lane) & (kGvRing - 1)], row0);
    if (lane < et - eh) gv_consume<1, BATCH, GAIN, XS>(a, S, xs, ring_even[(eh + lane) & (kGvRing - 1)], row0);
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicOr(flags, kFlagIndexRange);
}

}  // namespace llvq
