// bwd.cuh -- backward of the fused BitLinear layer with the straight-through
// estimator (ld246.com, section "训练与优化：新的策略": the non-differentiable
// ternary weights and quantisation are back-propagated with a surrogate
// gradient, read as passing gradients through the quantisers unchanged).
// With x_q = q * (absmax / 127) and W_q = w~ * beta the forward is
// y = x_q . W_q^T, so
//   dr = dy . W_q            (the gradient at the normalised activations)
//   dW = dy^T . x_q          (the gradient at the latent weights)
// and RMSNorm's backward gives dx and dgamma from dr.  The two products are
// plain bf16 GEMMs (cuBLAS, fp32 accumulation) over operands these kernels
// prepare: w~ as bf16 {-1, 0, +1} (beta is applied to dr afterwards, exactly),
// q as bf16 (exact) and dy * absmax / 127 rounded to bf16.
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kBwdThreads = 256;

// w~ as bf16 from the packed codes: one thread per 32-bit word (16 weights)
__global__ void __launch_bounds__(kBwdThreads) unpack_ternary_bf16_kernel(const uint32_t* __restrict__ packed,
                                                                          int64_t nwords,
                                                                          uint16_t* __restrict__ wb) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kBwdThreads + threadIdx.x;
    if (i >= nwords) return;
    const uint32_t w = __ldg(packed + i);
    // weight j of the group: code at bits 8 (j % 4) + 2 (j / 4); bf16 of c - 1
    uint32_t out[8];
#pragma unroll
    for (int j2 = 0; j2 < 8; ++j2) {
        uint32_t pair = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = 2 * j2 + h;
            const uint32_t c = (w >> (8 * (j & 3) + 2 * (j >> 2))) & 3u;
            const uint32_t bits = c == 0 ? 0xBF80u : (c == 2 ? 0x3F80u : 0u);  // -1, +1, 0
            pair |= bits << (16 * h);
        }
        out[j2] = pair;
    }
    uint4* dst = reinterpret_cast<uint4*>(wb + 16 * i);
    dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
    dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
}

// dy * (absmax / 127) as bf16 (the left operand of dW), one thread per element
__global__ void __launch_bounds__(kBwdThreads) scale_dy_kernel(const uint16_t* __restrict__ dy,
                                                               const float* __restrict__ absmax, int64_t M, int64_t N,
                                                               uint16_t* __restrict__ dys) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kBwdThreads + threadIdx.x;
    if (i >= M * N) return;
    const int64_t m = i / N;
    const float s = __fdiv_rn(__ldg(absmax + m), 127.0f);
    const float v = __fmul_rn(__uint_as_float(static_cast<uint32_t>(__ldg(dy + i)) << 16), s);
    dys[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// q as bf16 (exact for |q| <= 127), one thread per element
__global__ void __launch_bounds__(kBwdThreads) codes_bf16_kernel(const int8_t* __restrict__ q, int64_t n,
                                                                 uint16_t* __restrict__ qb) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kBwdThreads + threadIdx.x;
    if (i >= n) return;
    qb[i] = __bfloat16_as_ushort(__float2bfloat16_rn(static_cast<float>(__ldg(q + i))));
}

// RMSNorm backward for one token row per CTA: with g_k = beta * dr_k,
//   dx_k = inv gamma_k g_k - x_k inv^3 (sum_j gamma_j g_j x_j) / K
// inv recomputed as 1 / sqrt(sum x^2 / K + eps) (fp64 sums; fixed-order
// reductions); also writes inv per row for the dgamma column sums.
__global__ void __launch_bounds__(kBwdThreads) rmsnorm_bwd_kernel(const uint16_t* __restrict__ x,
                                                                  const float* __restrict__ gamma,
                                                                  const float* __restrict__ dr,
                                                                  const float* __restrict__ beta, float eps, int K,
                                                                  uint16_t* __restrict__ dx,
                                                                  float* __restrict__ inv_out) {
    __shared__ double red_a[kBwdThreads / 32], red_b[kBwdThreads / 32];
    const int64_t m = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint16_t* xr = x + m * static_cast<int64_t>(K);
    const float* dr_r = dr + m * static_cast<int64_t>(K);
    const double bt = static_cast<double>(__ldg(beta));
    double s2 = 0.0, dot = 0.0;
    for (int k = threadIdx.x; k < K; k += kBwdThreads) {
        const double xv = __uint_as_float(static_cast<uint32_t>(__ldg(xr + k)) << 16);
        s2 += xv * xv;
        dot += static_cast<double>(__ldg(gamma + k)) * (bt * static_cast<double>(__ldg(dr_r + k))) * xv;
    }
    s2 = warp_sum_f64(s2);
    dot = warp_sum_f64(dot);
    if (lane == 0) {
        red_a[warp] = s2;
        red_b[warp] = dot;
    }
    __syncthreads();
    s2 = 0.0;
    dot = 0.0;
#pragma unroll
    for (int w = 0; w < kBwdThreads / 32; ++w) {
        s2 += red_a[w];
        dot += red_b[w];
    }
    const double inv = 1.0 / sqrt(s2 / static_cast<double>(K) + static_cast<double>(eps));
    const double c2 = inv * inv * inv * dot / static_cast<double>(K);
    for (int k = threadIdx.x; k < K; k += kBwdThreads) {
        const double xv = __uint_as_float(static_cast<uint32_t>(__ldg(xr + k)) << 16);
        const double g = inv * static_cast<double>(__ldg(gamma + k)) * (bt * static_cast<double>(__ldg(dr_r + k))) -
                         xv * c2;
        dx[m * static_cast<int64_t>(K) + k] = __bfloat16_as_ushort(__double2bfloat16(g));
    }
    if (threadIdx.x == 0) inv_out[m] = static_cast<float>(inv);
}

// dgamma_k = beta * sum_m dr[m][k] x[m][k] inv_m, in two deterministic
// stages: partial sums over chunks of kDgammaRows rows (one thread per column,
// rows in order, fp64), then each column's partials in chunk order.
constexpr int kDgammaRows = 64;

__global__ void __launch_bounds__(kBwdThreads) dgamma_partial_kernel(const uint16_t* __restrict__ x,
                                                                     const float* __restrict__ dr,
                                                                     const float* __restrict__ inv, int64_t M, int K,
                                                                     double* __restrict__ part) {
    const int k = blockIdx.x * kBwdThreads + threadIdx.x;
    if (k >= K) return;
    const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kDgammaRows;
    const int64_t m1 = m0 + kDgammaRows < M ? m0 + kDgammaRows : M;
    double s = 0.0;
    for (int64_t m = m0; m < m1; ++m) {
        const double xv = __uint_as_float(static_cast<uint32_t>(__ldg(x + m * K + k)) << 16);
        s += static_cast<double>(__ldg(dr + m * K + k)) * xv * static_cast<double>(__ldg(inv + m));
    }
    part[static_cast<int64_t>(blockIdx.y) * K + k] = s;
}

__global__ void __launch_bounds__(kBwdThreads) dgamma_final_kernel(const double* __restrict__ part, int chunks, int K,
                                                                   const float* __restrict__ beta,
                                                                   float* __restrict__ dgamma) {
    const int k = blockIdx.x * kBwdThreads + threadIdx.x;
    if (k >= K) return;
    double s = 0.0;
    for (int c = 0; c < chunks; ++c) s += part[static_cast<int64_t>(c) * K + k];
    dgamma[k] = static_cast<float>(s * static_cast<double>(__ldg(beta)));
}

}  // namespace mmf
