// gptq48.cuh -- one pass of Spherical GPTQ over a weight matrix on the 48-bit union (kernels; the
// host loop is llvq_spherical_gptq in llvq.cu).
//
// "Leech Lattice Vector Quantization for Efficient LLM Compression", papernotes.org notes,
// 方法详解 / 关键设计 3 (保模长球面曲率反馈): the shape-gain candidate w~ is rescaled to the
// original norm, w^ = (|w| / |w~|) w~ -- a retraction onto the product of spheres -- and the
// residual E = w - w^ is propagated to the weights not yet quantized through U = chol(H^-1)^T.
// Per 24-column block B, in column order, every row's block is quantized jointly: its direction
// v is the angular search over the union of the block rounded to fp32, so w^ = |w| v / |v|, and
// the later columns move by -E G_B with G_B = U_BB^-1 U_B,rest (GPTQ's per-column update
// -e / U_ii U_i,rest in block form: the inverse Hessian of the columns left is the trailing block
// of U^T U).
//
// Every step is fp64 in one fixed operation order, the same as the CPU oracle's, so that the two
// agree bit for bit: |w|^2 as an fma chain over i ascending; ratio = sqrt(|w|^2) / sqrt(16 m);
// w^_i = ratio v_i; G_B by back substitution per column, g_i = (u_i + sum_{k>i} (-U_ik) g_k) / U_ii
// with the sum an fma chain over k ascending starting from u_i; each later weight
// W -= (fma chain over k ascending of E_k G_B[k][c], starting from 0); no other product is fused
// into an addition.
#pragma once
#include <cstdint>

namespace llvq {

constexpr int kGqThreads = 256;

// G [nb][24][cols]: block b's rows at [b][k][c] for c >= 24 (b + 1) (other columns untouched).
// Grid (ceil(cols / kGqThreads), nb): thread = one column of one block.
__global__ void __launch_bounds__(kGqThreads) k_gptq_gmat(const double *__restrict__ U, double *__restrict__ G,
                                                          int cols) {
    __shared__ double ubb[24][24];
    const int b = blockIdx.y, base = 24 * b;
    for (int t = threadIdx.x; t < 24 * 24; t += blockDim.x)
        ubb[t / 24][t % 24] = U[(size_t)(base + t / 24) * cols + base + t % 24];
    __syncthreads();
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c < base + 24 || c >= cols) return;
    double g[24];
#pragma unroll
    for (int i = 23; i >= 0; i--) {
        double acc = U[(size_t)(base + i) * cols + c];
#pragma unroll
        for (int k = i + 1; k < 24; k++) acc = fma(-ubb[i][k], g[k], acc);
        g[i] = acc / ubb[i][i];
    }
    double *out = G + (size_t)b * 24 * cols + c;
#pragma unroll
    for (int i = 0; i < 24; i++) out[(size_t)i * cols] = g[i];
}

// Xf [rows][24] = fp32(W[:, 24 b .. 24 b + 23]) (round to nearest), the search's input.
__global__ void k_gptq_gather(const double *__restrict__ W, float *__restrict__ Xf, int rows, int cols, int b) {
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (long long)rows * 24) return;
    const long long r = t / 24;
    const int i = (int)(t % 24);
    Xf[t] = (float)W[r * cols + 24 * b + i];
}

// One thread per row: the retraction of the row's block onto |w| v / |v|, its residual E [rows][24],
// the block written back as w^, the point and the norm recorded.
__global__ void k_gptq_retract(double *__restrict__ W, const int8_t *__restrict__ P, double *__restrict__ E,
                               int8_t *__restrict__ points, double *__restrict__ norms, int rows, int cols, int b) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const int nb = cols / 24;
    double *w = W + (size_t)r * cols + 24 * b;
    double s = 0.0;
    int n2 = 0;
    int v[24];
#pragma unroll
    for (int i = 0; i < 24; i++) {
        v[i] = P[(size_t)r * 24 + i];
        s = fma(w[i], w[i], s);
        n2 += v[i] * v[i];
    }
    const double ratio = sqrt(s) / sqrt((double)n2);
#pragma unroll
    for (int i = 0; i < 24; i++) {
        const double what = __dmul_rn(ratio, (double)v[i]);   // _rn: never fused with the subtraction
        E[(size_t)r * 24 + i] = __dsub_rn(w[i], what);
        w[i] = what;
        points[((size_t)r * nb + b) * 24 + i] = (int8_t)v[i];
    }
    norms[(size_t)r * nb + b] = sqrt(s);
}

// W[r][c] -= sum_k E[r][k] G_b[k][c] for the columns after block b.  Grid (ceil(rest / 256), rows):
// a CTA is one row (its 24 residuals in shared memory) and 256 consecutive columns.
__global__ void __launch_bounds__(kGqThreads) k_gptq_update(double *__restrict__ W, const double *__restrict__ E,
                                                            const double *__restrict__ G, int cols, int b) {
    __shared__ double e[24];
    const int r = blockIdx.y;
    if (threadIdx.x < 24) e[threadIdx.x] = E[(size_t)r * 24 + threadIdx.x];
    __syncthreads();
    const int c = 24 * (b + 1) + blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= cols) return;
    const double *g = G + (size_t)b * 24 * cols + c;
    double acc = 0.0;
#pragma unroll
    for (int k = 0; k < 24; k++) acc = fma(e[k], g[(size_t)k * cols], acc);
    W[(size_t)r * cols + c] -= acc;
}

}  // namespace llvq
