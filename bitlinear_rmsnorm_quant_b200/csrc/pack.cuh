// pack.cuh -- absmean ternarisation and 2-bit packing of latent weights
// (the absmean quantiser of the MatMul-free LM: datacamp.com, section "Thay
// MatMul bằng các phép toán tam phân").
//
// Three stream-ordered launches, all HBM-streaming:
//   1. absmean_partials: fixed grid, each block sums |W| over a fixed range in
//      fp64 with a fixed thread order and tree -> one double per block.  The
//      partials are written into the front of the `packed` output buffer,
//      which is not needed until step 3.
//   2. absmean_finalize: one block adds the partials in a fixed tree order,
//      divides by N*K in fp64, rounds once to fp32 -> scale[0].
//   3. ternary_encode: one thread per 16 weights: 64 B of fp32 in, one uint32
//      of 2-bit codes out (4 B read + 0.25 B written per weight).
// The grid of step 1 depends only on N*K, so beta is bit-identical run to run.
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kPackThreads = 256;

// Number of fp64 partials for n weights: one per 64 Ki weights, at most 2048;
// always fits in the packed buffer (n/4 bytes >= 8 bytes per partial).
__host__ __device__ inline int absmean_num_partials(int64_t n) {
    int64_t p = n >> 16;
    if (p < 1) p = 1;
    if (p > 2048) p = 2048;
    return static_cast<int>(p);
}

__device__ __forceinline__ double block_sum_f64(double v, double* red /* [kPackThreads/32] */) {
    v = warp_sum_f64(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double s = 0.0;
    if (warp == 0) {
        s = (lane < kPackThreads / 32) ? red[lane] : 0.0;
        s = warp_sum_f64(s);
    }
    return s;  // valid in warp 0
}

// Block b sums |W[i]| for i in [b*chunk, min(n, (b+1)*chunk)), chunk a multiple
// of 4; thread t takes float4 groups t, t+T, ... of that range.
__global__ void __launch_bounds__(kPackThreads) absmean_partials_kernel(const float* __restrict__ W, int64_t n,
                                                                        int64_t chunk, double* __restrict__ partials) {
    __shared__ double red[kPackThreads / 32];
    const int64_t begin = static_cast<int64_t>(blockIdx.x) * chunk;
    const int64_t end = min(n, begin + chunk);
    double s = 0.0;
    const float4* W4 = reinterpret_cast<const float4*>(W);
    for (int64_t g = begin / 4 + threadIdx.x; g < end / 4; g += kPackThreads) {
        const float4 v = __ldg(W4 + g);
        s += fabs(static_cast<double>(v.x)) + fabs(static_cast<double>(v.y));
        s += fabs(static_cast<double>(v.z)) + fabs(static_cast<double>(v.w));
    }
    s = block_sum_f64(s, red);
    if (threadIdx.x == 0) partials[blockIdx.x] = s;
}

__global__ void __launch_bounds__(kPackThreads) absmean_finalize_kernel(const double* __restrict__ partials,
                                                                        int np, int64_t n, float* __restrict__ scale) {
    __shared__ double red[kPackThreads / 32];
    double s = 0.0;
    for (int i = threadIdx.x; i < np; i += kPackThreads) s += partials[i];
    s = block_sum_f64(s, red);
    if (threadIdx.x == 0) scale[0] = static_cast<float>(s / static_cast<double>(n));
}

// One thread per packed word (16 consecutive weights of a row; rows are
// contiguous, so word w covers weights 16w .. 16w+15 of the flat matrix).
__global__ void __launch_bounds__(kPackThreads) ternary_encode_kernel(const float* __restrict__ W, int64_t nwords,
                                                                      float eps_w, const float* __restrict__ scale,
                                                                      uint32_t* __restrict__ packed) {
    const float d = __fadd_rn(__ldg(scale), eps_w);
    const float4* W4 = reinterpret_cast<const float4*>(W);
    for (int64_t w = static_cast<int64_t>(blockIdx.x) * kPackThreads + threadIdx.x; w < nwords;
         w += static_cast<int64_t>(gridDim.x) * kPackThreads) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {           // weights 4j .. 4j+3 of the group
            const float4 v = __ldg(W4 + 4 * w + j);
            const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int b = 0; b < 4; ++b) {       // weight i = 4j + b -> byte b, bits 2j
                const float t = rintf(__fdiv_rn(e[b], d));
                const uint32_t code = t > 0.5f ? 2u : (t < -0.5f ? 0u : 1u);
                word |= code << (8 * b + 2 * j);
            }
        }
        packed[w] = word;
    }
}

}  // namespace mmf
