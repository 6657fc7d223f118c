// quant.cuh -- fused RMSNorm + per-token absmax int8 quantisation for the
// large-M path (RMSNorm before quantisation: datacamp.com, component figure,
// item "RMS norm"; fused so x is read from HBM once: ld246.com, section
// "融合 BitLinear 层的创新").
//
// One CTA per token row.  The row is streamed from HBM once into shared memory
// (16-byte loads), then:
//   ms  = (float)(sum x^2 / K)         fp64 sum (bf16 squares are exact in fp64)
//   inv = 1 / sqrt(ms + eps)           fp32, correctly rounded
//   r   = (x * inv) * gamma            fp32, two roundings
//   a   = max(max |r|, 1e-5); s = 127 / a
//   q   = clamp(rint(r * s), -127, 127)
// and writes q (int8 [M][K]), absmax a, and qsum = sum_k q (used by the
// contraction kernels, which work with codes w~ + 1 and subtract qsum).
// HBM traffic per element: 2 B read + 1 B written.
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kQuantThreads = 256;

template <typename T, typename Op>
__device__ __forceinline__ T block_allreduce(T v, T* red /* [kQuantThreads/32 + 1] */, Op op) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        T s = red[lane < kQuantThreads / 32 ? lane : 0];
        if (lane >= kQuantThreads / 32) s = T(0);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s = op(s, __shfl_xor_sync(0xffffffffu, s, o));
        if (lane == 0) red[kQuantThreads / 32] = s;
    }
    __syncthreads();
    const T out = red[kQuantThreads / 32];
    __syncthreads();  // red may be reused by the next reduction
    return out;
}

struct AddOp {
    template <typename T>
    __device__ __forceinline__ T operator()(T a, T b) const { return a + b; }
};
struct MaxOp {
    __device__ __forceinline__ float operator()(float a, float b) const { return fmaxf(a, b); }
};

// 8 bf16 in a uint4 -> 8 floats
__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__global__ void __launch_bounds__(kQuantThreads) rmsnorm_quant_kernel(const uint16_t* __restrict__ x,
                                                                      const float* __restrict__ gamma, float eps,
                                                                      int K, int8_t* __restrict__ q,
                                                                      float* __restrict__ absmax,
                                                                      int* __restrict__ qsum) {
    extern __shared__ uint4 xs[];  // K/8 chunks of 8 bf16
    __shared__ double red_d[kQuantThreads / 32 + 1];
    __shared__ float red_f[kQuantThreads / 32 + 1];
    __shared__ int red_i[kQuantThreads / 32 + 1];

    pdl_wait();  // x may come from the previous kernel (no-op unless launched as a dependent)
    pdl_launch_dependents();
    const int64_t m = blockIdx.x;
    const int C = K >> 3;
    const uint4* xr = reinterpret_cast<const uint4*>(x + m * static_cast<int64_t>(K));
    const float4* g4 = reinterpret_cast<const float4*>(gamma);

    double s2 = 0.0;
    for (int c = threadIdx.x; c < C; c += kQuantThreads) {
        const uint4 v = __ldcs(xr + c);  // streamed once: evict-first
        xs[c] = v;
        float f[8];
        unpack_bf16x8(v, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) s2 += static_cast<double>(f[i]) * static_cast<double>(f[i]);
    }
    s2 = block_allreduce(s2, red_d, AddOp());
    const float ms = static_cast<float>(s2 / static_cast<double>(K));
    const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));

    float amax = 0.0f;
    for (int c = threadIdx.x; c < C; c += kQuantThreads) {
        float f[8];
        unpack_bf16x8(xs[c], f);
        const float4 ga = __ldg(g4 + 2 * c), gb = __ldg(g4 + 2 * c + 1);
        const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(__fmul_rn(__fmul_rn(f[i], inv), g[i])));
    }
    amax = block_allreduce(amax, red_f, MaxOp());
    const float a = fmaxf(amax, 1e-5f);
    const float s = __fdiv_rn(127.0f, a);

    int qs = 0;
    uint2* qr = reinterpret_cast<uint2*>(q + m * static_cast<int64_t>(K));
    for (int c = threadIdx.x; c < C; c += kQuantThreads) {
        float f[8];
        unpack_bf16x8(xs[c], f);
        const float4 ga = __ldg(g4 + 2 * c), gb = __ldg(g4 + 2 * c + 1);
        const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int code = quant_code(__fmul_rn(__fmul_rn(f[i], inv), g[i]), s);
            qs += code;
            packed[i >> 2] |= (static_cast<uint32_t>(code) & 0xFFu) << (8 * (i & 3));
        }
        __stcs(qr + c, make_uint2(packed[0], packed[1]));
    }
    qs = block_allreduce(qs, red_i, AddOp());
    if (threadIdx.x == 0) {
        absmax[m] = a;
        if (qsum) qsum[m] = qs;
    }
}

// qsum only (for the contraction alone, when q is given).
__global__ void __launch_bounds__(kQuantThreads) qsum_kernel(const int8_t* __restrict__ q, int K,
                                                             int* __restrict__ qsum) {
    __shared__ int red_i[kQuantThreads / 32 + 1];
    const int64_t m = blockIdx.x;
    const uint4* qr = reinterpret_cast<const uint4*>(q + m * static_cast<int64_t>(K));
    int s = 0;
    for (int c = threadIdx.x; c < (K >> 4); c += kQuantThreads) {
        const uint4 v = __ldg(qr + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) s += __dp4a(static_cast<int>(w[i]), 0x01010101, 0);
    }
    s = block_allreduce(s, red_i, AddOp());
    if (threadIdx.x == 0) qsum[m] = s;
}

}  // namespace mmf
