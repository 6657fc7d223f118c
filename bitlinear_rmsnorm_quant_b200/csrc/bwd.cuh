// bwd.cuh -- the parts of the straight-through backward of the fused
// BitLinear layer around its two products (ld246.com, section "训练与优化：新的
// 策略": the non-differentiable ternary weights and quantisation are
// back-propagated with a surrogate gradient, read as passing gradients through
// the quantisers unchanged).  With x_q = q * (absmax / 127) and
// W_q = w~ * beta the forward is y = x_q . W_q^T, so
//   dr = dy . W_q            (the gradient at the normalised activations)
//   dW = dy^T . x_q          (the gradient at the latent weights)
// (both on the tensor cores, bwd_tc.cuh), and RMSNorm's backward gives dx and
// dgamma from dr (here).
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kBwdThreads = 256;

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
