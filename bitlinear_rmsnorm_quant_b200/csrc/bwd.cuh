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

// Final dgamma stage: a CTA takes 32 columns; its 32 warps sum the partials
// of chunks w, w + 32, w + 64, ... in order (one column per lane, 256-byte
// rows per warp), then warp 0 adds the 32 group sums in warp order.
constexpr int kDgCols = 32;
constexpr int kDgThreads = 1024;
constexpr int kDgGroups = kDgThreads / kDgCols;

__global__ void __launch_bounds__(kDgThreads) dgamma_final_kernel(const double* __restrict__ part, int chunks, int K,
                                                                   const float* __restrict__ beta,
                                                                   float* __restrict__ dgamma) {
    __shared__ double red[kDgGroups][kDgCols];
    const int col = threadIdx.x & (kDgCols - 1), grp = threadIdx.x / kDgCols;
    const int k = blockIdx.x * kDgCols + col;
    double s = 0.0;
    if (k < K) {
#pragma unroll 8
        for (int c = grp; c < chunks; c += kDgGroups) s += __ldg(part + static_cast<int64_t>(c) * K + k);
    }
    red[grp][col] = s;
    __syncthreads();
    if (grp == 0 && k < K) {
        double t = 0.0;
#pragma unroll
        for (int g = 0; g < kDgGroups; ++g) t += red[g][col];
        dgamma[k] = static_cast<float>(t * static_cast<double>(__ldg(beta)));
    }
}

// RMSNorm backward and the dgamma partial sums in one pass over HBM (K <=
// 8192): a CTA takes kBwdFusedRows consecutive token rows, RPB rows per
// barrier; thread t owns the 8-column chunks c = t + 256 i (i < CPT), holds
// their x and dr in registers for the row, and keeps its columns' dgamma
// partial sums over the CTA's rows.  Per row the sums of x^2 and gamma dr x
// are fp32 over a thread's columns (x^2 of a bf16 value is exact in fp32),
// fp64 across the threads (a warp tree, then the warps in index order), and
// inv, c2 fp64; dx and the partials are formed in fp32 (dx is rounded to bf16
// once at the end).  The CTA's partials go to part[blockIdx.x][k] (fp64);
// dgamma_final_kernel sums them over the CTAs in order.
constexpr int kBwdFusedRows = 16;
constexpr int kBwdFusedMaxK = kBwdThreads * 8 * 4;

template <int CPT, int RPB>
__global__ void __launch_bounds__(kBwdThreads) rmsnorm_bwd_fused_kernel(const uint16_t* __restrict__ x,
                                                                        const float* __restrict__ gamma,
                                                                        const float* __restrict__ dr,
                                                                        const float* __restrict__ beta, float eps,
                                                                        int K, int64_t M,
                                                                        uint16_t* __restrict__ dx,
                                                                        double* __restrict__ part) {
    __shared__ double red[2][RPB][2][kBwdThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = K >> 3;
    const double bt = static_cast<double>(__ldg(beta));
    const float4* g4 = reinterpret_cast<const float4*>(gamma);
    float acc[CPT][8];
#pragma unroll
    for (int i = 0; i < CPT; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i][e] = 0.0f;
    const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kBwdFusedRows;
    const int64_t m1 = m0 + kBwdFusedRows < M ? m0 + kBwdFusedRows : M;
    for (int64_t m = m0; m < m1; m += RPB) {
        const int buf = static_cast<int>((m - m0) / RPB) & 1;
        uint4 xw[RPB][CPT];
        float4 da[RPB][CPT], db[RPB][CPT];
#pragma unroll
        for (int r = 0; r < RPB; ++r)
#pragma unroll
            for (int i = 0; i < CPT; ++i) {
                const int c = threadIdx.x + kBwdThreads * i;
                if (c < C && m + r < m1) {
                    const int64_t off = (m + r) * static_cast<int64_t>(K) + 8 * c;
                    xw[r][i] = __ldg(reinterpret_cast<const uint4*>(x + off));
                    da[r][i] = __ldg(reinterpret_cast<const float4*>(dr + off));
                    db[r][i] = __ldg(reinterpret_cast<const float4*>(dr + off) + 1);
                } else {
                    xw[r][i] = make_uint4(0u, 0u, 0u, 0u);
                    da[r][i] = db[r][i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                }
            }
#pragma unroll
        for (int r = 0; r < RPB; ++r) {
            float s2 = 0.0f, dot = 0.0f;
#pragma unroll
            for (int i = 0; i < CPT; ++i) {
                const int c = threadIdx.x + kBwdThreads * i;
                if (c < C) {
                    float xv[8];
                    unpack_bf16x8(xw[r][i], xv);
                    const float4 ga = __ldg(g4 + 2 * c), gb = __ldg(g4 + 2 * c + 1);
                    const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                    const float d[8] = {da[r][i].x, da[r][i].y, da[r][i].z, da[r][i].w,
                                        db[r][i].x, db[r][i].y, db[r][i].z, db[r][i].w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        s2 = fmaf(xv[e], xv[e], s2);
                        dot = fmaf(g[e] * d[e], xv[e], dot);
                    }
                }
            }
            const double s2w = warp_sum_f64(static_cast<double>(s2));
            const double dotw = warp_sum_f64(static_cast<double>(dot));
            if (lane == 0) {
                red[buf][r][0][warp] = s2w;
                red[buf][r][1][warp] = dotw;
            }
        }
        __syncthreads();  // (the other buffer was last read before the previous barrier)
#pragma unroll
        for (int r = 0; r < RPB; ++r) {
            double s2 = 0.0, dot = 0.0;
#pragma unroll
            for (int w = 0; w < kBwdThreads / 32; ++w) {
                s2 += red[buf][r][0][w];
                dot += red[buf][r][1][w];
            }
            const double inv = 1.0 / sqrt(s2 / static_cast<double>(K) + static_cast<double>(eps));
            const float c2 = static_cast<float>(inv * inv * inv * (bt * dot) / static_cast<double>(K));
            const float ib = static_cast<float>(inv * bt), invf = static_cast<float>(inv);
            if (m + r < m1) {
#pragma unroll
                for (int i = 0; i < CPT; ++i) {
                    const int c = threadIdx.x + kBwdThreads * i;
                    if (c < C) {
                        float xv[8];
                        unpack_bf16x8(xw[r][i], xv);
                        const float4 ga = __ldg(g4 + 2 * c), gb = __ldg(g4 + 2 * c + 1);
                        const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                        const float d[8] = {da[r][i].x, da[r][i].y, da[r][i].z, da[r][i].w,
                                            db[r][i].x, db[r][i].y, db[r][i].z, db[r][i].w};
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float v0 = fmaf(ib * g[2 * e], d[2 * e], -xv[2 * e] * c2);
                            const float v1 = fmaf(ib * g[2 * e + 1], d[2 * e + 1], -xv[2 * e + 1] * c2);
                            const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
                            o[e] = *reinterpret_cast<const uint32_t*>(&h);
                            acc[i][2 * e] = fmaf(d[2 * e] * xv[2 * e], invf, acc[i][2 * e]);
                            acc[i][2 * e + 1] = fmaf(d[2 * e + 1] * xv[2 * e + 1], invf, acc[i][2 * e + 1]);
                        }
                        *reinterpret_cast<uint4*>(dx + (m + r) * static_cast<int64_t>(K) + 8 * c) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = threadIdx.x + kBwdThreads * i;
        if (c < C) {
            double* pr = part + static_cast<int64_t>(blockIdx.x) * K + 8 * c;
#pragma unroll
            for (int e = 0; e < 8; ++e) pr[e] = static_cast<double>(acc[i][e]);
        }
    }
}

}  // namespace mmf
