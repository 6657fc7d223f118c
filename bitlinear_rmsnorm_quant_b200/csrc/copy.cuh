// copy.cuh -- streaming 128-bit device-to-device copy.  Measurement kernel:
// its achieved read+write bandwidth is the HBM roofline stated beside the
// BitLinear kernels' fractions.
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kCopyThreads = 512;
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(kCopyThreads) hbm_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                                int64_t n16) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kCopyThreads;
    int64_t i = static_cast<int64_t>(blockIdx.x) * kCopyThreads + threadIdx.x;
    for (; i + (kCopyUnroll - 1) * stride < n16; i += kCopyUnroll * stride) {
        uint4 v[kCopyUnroll];
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) v[u] = __ldcs(src + i + u * stride);
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) __stcs(dst + i + u * stride, v[u]);
    }
    for (; i < n16; i += stride) __stcs(dst + i, __ldcs(src + i));
}

}  // namespace mmf
