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

// RMSNorm backward and the dgamma partial sums in one pass over HBM (K <=
// 8192): a CTA takes kBwdFusedRows consecutive token rows; thread t owns the
// 8-column chunks c = t + 256 i (i < CPT) and keeps its columns' dgamma
// partial sums (fp64) in registers over the CTA's rows.  Per row it reads x
// and dr (16- and 32-byte loads, kept in L1), forms the row's fp64 sums of
// x^2 and gamma beta dr x (a warp tree, then the warps in index order), then
// reads the same lines again from L1 to write dx and add dr x inv to its
// partials, rows in order.  The CTA's partials go to part[blockIdx.x][k];
// dgamma_final_kernel sums them over the CTAs in order.
constexpr int kBwdFusedRows = 16;
constexpr int kBwdFusedMaxK = kBwdThreads * 8 * 4;

__device__ __forceinline__ void load_x8_dr8(const uint16_t* x, const float* dr, int64_t off, float (&xv)[8],
                                            float (&dv)[8]) {
    const uint4 xw = __ldg(reinterpret_cast<const uint4*>(x + off));
    const float4 da = __ldg(reinterpret_cast<const float4*>(dr + off));
    const float4 db = __ldg(reinterpret_cast<const float4*>(dr + off) + 1);
    const uint32_t w[4] = {xw.x, xw.y, xw.z, xw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        xv[2 * e] = __uint_as_float(w[e] << 16);
        xv[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
    dv[0] = da.x; dv[1] = da.y; dv[2] = da.z; dv[3] = da.w;
    dv[4] = db.x; dv[5] = db.y; dv[6] = db.z; dv[7] = db.w;
}

template <int CPT>
__global__ void __launch_bounds__(kBwdThreads) rmsnorm_bwd_fused_kernel(const uint16_t* __restrict__ x,
                                                                        const float* __restrict__ gamma,
                                                                        const float* __restrict__ dr,
                                                                        const float* __restrict__ beta, float eps,
                                                                        int K, int64_t M,
                                                                        uint16_t* __restrict__ dx,
                                                                        double* __restrict__ part) {
    __shared__ double red_s[2][kBwdThreads / 32], red_d[2][kBwdThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = K >> 3;
    const double bt = static_cast<double>(__ldg(beta));
    const float4* g4 = reinterpret_cast<const float4*>(gamma);
    double acc[CPT][8];
#pragma unroll
    for (int i = 0; i < CPT; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i][e] = 0.0;
    const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kBwdFusedRows;
    const int64_t m1 = m0 + kBwdFusedRows < M ? m0 + kBwdFusedRows : M;
    for (int64_t m = m0; m < m1; ++m) {
        const int buf = static_cast<int>(m - m0) & 1;
        const int64_t row = m * static_cast<int64_t>(K);
        double s2 = 0.0, dot = 0.0;
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = threadIdx.x + kBwdThreads * i;
            if (c < C) {
                float xv[8], dv[8];
                load_x8_dr8(x, dr, row + 8 * c, xv, dv);
                const float4 ga = __ldg(g4 + 2 * c), gb = __ldg(g4 + 2 * c + 1);
                const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const double xd = xv[e];
                    s2 += xd * xd;
                    dot += static_cast<double>(g[e]) * (bt * static_cast<double>(dv[e])) * xd;
                }
            }
        }
        s2 = warp_sum_f64(s2);
        dot = warp_sum_f64(dot);
        if (lane == 0) {
            red_s[buf][warp] = s2;
            red_d[buf][warp] = dot;
        }
        __syncthreads();  // (the other buffer was last read before the previous row's barrier)
        s2 = 0.0;
        dot = 0.0;
#pragma unroll
        for (int w = 0; w < kBwdThreads / 32; ++w) {
            s2 += red_s[buf][w];
            dot += red_d[buf][w];
        }
        const double inv = 1.0 / sqrt(s2 / static_cast<double>(K) + static_cast<double>(eps));
        const double c2 = inv * inv * inv * dot / static_cast<double>(K);
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = threadIdx.x + kBwdThreads * i;
            if (c < C) {
                float xv[8], dv[8];
                load_x8_dr8(x, dr, row + 8 * c, xv, dv);
                const float4 ga = __ldg(g4 + 2 * c), gb = __ldg(g4 + 2 * c + 1);
                const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    uint32_t h[2];
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int k = 2 * e + j;
                        const double xd = xv[k], drd = static_cast<double>(dv[k]);
                        const double gr = inv * static_cast<double>(g[k]) * (bt * drd) - xd * c2;
                        h[j] = __bfloat16_as_ushort(__double2bfloat16(gr));
                        acc[i][k] += drd * xd * inv;
                    }
                    o[e] = h[0] | (h[1] << 16);
                }
                *reinterpret_cast<uint4*>(dx + row + 8 * c) = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = threadIdx.x + kBwdThreads * i;
        if (c < C) {
            double* pr = part + static_cast<int64_t>(blockIdx.x) * K + 8 * c;
#pragma unroll
            for (int e = 0; e < 8; ++e) pr[e] = acc[i][e];
        }
    }
}

}  // namespace mmf
