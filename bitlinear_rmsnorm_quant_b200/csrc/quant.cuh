// quant.cuh -- fused RMSNorm + per-token absmax int8 quantisation for the
// large-M path (RMSNorm before quantisation: datacamp.com, component figure,
// item "RMS norm"; fused so x is read from HBM once: ld246.com, section
// "融合 BitLinear 层的创新").
//
// Each token row is read from HBM once (for large M, a persistent kernel that
// keeps rows in registers, one to four warps per row; otherwise one 8-warp CTA
// per row with the row staged in shared memory), then:
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

// Byte offset of codes k = 8 c8 .. 8 c8 + 7 of token m in the decode
// tensor-core kernel's operand layout for NT token rows: per 128-wide K
// chunk, NT rows of 128 bytes in 8-row 1024-byte atoms, 16-byte units
// swizzled by the row within the atom (the 128-byte swizzle the MMA's
// shared-memory descriptor reads; the kernel copies a chunk's NT rows as the
// first rows of its A tile).
__host__ __device__ __forceinline__ int64_t blayout_offset(int64_t m, int c8, int NT) {
    const int kc = c8 >> 4, u = (c8 & 15) >> 1, h = c8 & 1;
    const int r = static_cast<int>(m & 7);
    return static_cast<int64_t>(kc) * NT * 128 + (m >> 3) * 1024 + r * 128 + ((u ^ r) << 4) + 8 * h;
}

// WPR = 8 warps per token row and one row per CTA (what the library launches:
// below 4096 rows, for K above the register kernel's limit, and in GLU mode),
// or WPR = 1, a row per warp.  One thread brings the whole row into shared memory with bulk
// copies (one request per row, so the row's HBM latency is paid once, not once
// per 16-byte load); the three passes then run from shared memory, reduced
// across the row's warps in index order.  With WPR = 1 a CTA holds one row per
// warp and needs no CTA-wide barrier.
constexpr int kQuantCtaWarps = 8;
constexpr uint32_t kQuantPieceBytes = 32 * 1024;  // bytes per bulk copy request
constexpr int64_t kQuantWarpRowMinM = 4096;       // rows from which the register kernel takes over

// GLU: x is the gate g of the GLU channel mixer and the row normalised is
// p = bf16(SiLU(g) * u), formed in pass 1 and kept in place of x.
// bl_nt > 0: the codes go to q in the operand layout of NT = bl_nt token rows
// (blayout_offset) for the decode tensor-core kernel; the grid then has
// bl_nt CTAs and those of rows M .. bl_nt - 1 write zero codes.
template <int WPR, bool GLU = false>
__global__ void __launch_bounds__(kQuantCtaWarps * 32) rmsnorm_quant_kernel(const uint16_t* __restrict__ x,
                                                                              const float* __restrict__ gamma,
                                                                              float eps, int K, int64_t M,
                                                                              int8_t* __restrict__ q,
                                                                              float* __restrict__ absmax,
                                                                              int* __restrict__ qsum,
                                                                              const uint16_t* __restrict__ u,
                                                                              int bl_nt) {
    // one row per CTA (WPR = 8: the reductions below share one set of slots)
    // or one row per warp (WPR = 1: warp reductions only)
    static_assert(WPR == 1 || WPR == kQuantCtaWarps, "one row per warp or one row per CTA");
    extern __shared__ __align__(128) uint4 xs_all[];  // one slice of K/8 chunks per row
    __shared__ __align__(8) uint64_t row_bar[kQuantCtaWarps];
    __shared__ double red_d[WPR];
    __shared__ float red_f[WPR];
    __shared__ int red_i[WPR];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rows = (blockDim.x >> 5) / WPR;
    const int rw = warp / WPR;  // row slot in the CTA
    const int wr = warp % WPR;  // warp within the row
    const int64_t m = static_cast<int64_t>(blockIdx.x) * rows + rw;
    if (wr == 0 && lane == 0) {
        mbar_init(&row_bar[rw], 1);
        mbar_fence_init();
    }
    if constexpr (WPR == 1) __syncwarp();
    else __syncthreads();
    pdl_wait();  // x may come from the previous kernel (no-op unless launched as a dependent)
    pdl_launch_dependents();
    const int C = K >> 3;
    if (m >= M) {  // WPR == 1: the whole warp; WPR > 1: only the padding rows of the operand layout
        if (bl_nt > 0 && m < bl_nt)
            for (int c = wr * 32 + lane; c < C; c += WPR * 32)
                *reinterpret_cast<uint2*>(q + blayout_offset(m, c, bl_nt)) = make_uint2(0u, 0u);
        return;
    }
    uint4* xs = xs_all + static_cast<size_t>(rw) * C;
    const uint8_t* xr = reinterpret_cast<const uint8_t*>(x + m * static_cast<int64_t>(K));
    const uint32_t row_bytes = static_cast<uint32_t>(K) * 2u;
    if (wr == 0 && lane == 0) {
        mbar_arrive_expect_tx(&row_bar[rw], row_bytes);
        for (uint32_t off = 0; off < row_bytes; off += kQuantPieceBytes) {
            const uint32_t n = row_bytes - off < kQuantPieceBytes ? row_bytes - off : kQuantPieceBytes;
            bulk_g2s(reinterpret_cast<uint8_t*>(xs) + off, xr + off, n, &row_bar[rw]);
        }
    }
    int abort_flag = 0;
    bool ok = mbar_wait(&row_bar[rw], 0, &abort_flag);
    if constexpr (WPR == 1) ok = __all_sync(0xffffffffu, ok);
    else ok = __syncthreads_and(ok);
    if (!ok) {
        int no_abort = 0;  // the copy may still be landing in this CTA's shared memory
        mbar_wait(&row_bar[rw], 0, &no_abort);
        return;
    }
    const float4* g4 = reinterpret_cast<const float4*>(gamma);
    const int c0 = wr * 32 + lane;
    constexpr int cstep = WPR * 32;

    // sum x^2: four fp64 chains per thread, a warp tree, then the row's warps in
    // index order (bf16 squares are exact in fp64)
    double s2[4] = {0.0, 0.0, 0.0, 0.0};
    for (int c = c0; c < C; c += cstep) {
        float f[8];
        if constexpr (GLU) {
            // this thread alone reads chunk c in the passes below
            const uint4 pv = glu_gate8(xs[c], __ldg(reinterpret_cast<const uint4*>(u + m * static_cast<int64_t>(K)) + c));
            xs[c] = pv;
            unpack_bf16x8(pv, f);
        } else {
            unpack_bf16x8(xs[c], f);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) s2[i & 3] += static_cast<double>(f[i]) * static_cast<double>(f[i]);
    }
    double s2w = warp_sum_f64((s2[0] + s2[1]) + (s2[2] + s2[3]));
    if constexpr (WPR > 1) {
        if (lane == 0) red_d[wr] = s2w;
        __syncthreads();
        s2w = red_d[0];
#pragma unroll
        for (int i = 1; i < WPR; ++i) s2w += red_d[i];
    }
    const float ms = static_cast<float>(s2w / static_cast<double>(K));
    const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));

    float amax[2] = {0.0f, 0.0f};
    for (int c = c0; c < C; c += cstep) {
        float f[8];
        unpack_bf16x8(xs[c], f);
        const float4 ga = __ldg(g4 + 2 * c), gb = __ldg(g4 + 2 * c + 1);
        const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
            amax[i & 1] = fmaxf(amax[i & 1], fabsf(__fmul_rn(__fmul_rn(f[i], inv), g[i])));
    }
    // amax >= 0, so its bits order like unsigned integers
    float amax_w = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(amax[0], amax[1]))));
    if constexpr (WPR > 1) {
        if (lane == 0) red_f[wr] = amax_w;
        __syncthreads();
        amax_w = red_f[0];
#pragma unroll
        for (int i = 1; i < WPR; ++i) amax_w = fmaxf(amax_w, red_f[i]);
    }
    const float a = fmaxf(amax_w, 1e-5f);
    const float s = __fdiv_rn(127.0f, a);

    int qs = 0;
    uint2* qr = reinterpret_cast<uint2*>(q + m * static_cast<int64_t>(K));
    for (int c = c0; c < C; c += cstep) {
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
        if (bl_nt > 0) *reinterpret_cast<uint2*>(q + blayout_offset(m, c, bl_nt)) = make_uint2(packed[0], packed[1]);
        else __stcs(qr + c, make_uint2(packed[0], packed[1]));
    }
    qs = __reduce_add_sync(0xffffffffu, qs);
    if constexpr (WPR > 1) {
        if (lane == 0) red_i[wr] = qs;
        __syncthreads();
        qs = red_i[0];
#pragma unroll
        for (int i = 1; i < WPR; ++i) qs += red_i[i];
    }
    if (wr == 0 && lane == 0) {
        absmax[m] = a;
        if (qsum) qsum[m] = qs;
    }
}

// Large M: a persistent grid of row groups; a group of WPR warps owns one row
// at a time and keeps it in registers (8 chunks of 8 bf16 per lane, so
// K <= 2048 * WPR), with the loads of its next row in flight while it works
// on the current one (two rows per lane in registers, no shared-memory
// staging of x; gamma is staged once per CTA).  Per row: the sum of squares
// in fp64 (exact for bf16 squares, so the order of the additions does not
// matter), the absmax of r = (x * inv) * gamma, then the codes.  A code is
// rounded by one float addition: in [2^23, 2^24) consecutive floats are 1
// apart, so adding 1.5 * 2^23 to v = r * s (|v| <= 127 up to one ulp, since
// s = 127 / a and a >= |r|) rounds v to the nearest integer, ties to even,
// and leaves it in the low byte (1.5 * 2^23 has a zero low byte).  The same
// integer as rint(v), which is already within [-127, 127], so the clamp of
// the definition never changes a code.  Four bytes are packed with byte
// permutes and summed with one DP4A.  The reductions are a fixed warp tree,
// then the group's warps in index order.
constexpr int kQuantRegChunks = 8;       // 16-byte chunks of x a lane holds per row (CHT), but 9 for three-warp rows
constexpr int kMaxQuantRegK = 8192;      // WPR <= 4

__host__ __device__ constexpr int quant_reg_warps(int WPR) { return WPR == 3 ? 6 : 8; }

template <int WPR, int CHT = 8>
__global__ void __launch_bounds__(quant_reg_warps(WPR) * 32, 2) rmsnorm_quant_reg_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ gamma, float eps, int K, int64_t M,
    int8_t* __restrict__ q, float* __restrict__ absmax, int* __restrict__ qsum) {
    constexpr int NW = quant_reg_warps(WPR);
    constexpr int RPC = NW / WPR;  // row groups per CTA
    constexpr int CH = CHT;
    extern __shared__ __align__(16) float4 gamma_s[];  // K / 4
    __shared__ double red_d[NW];
    __shared__ float red_f[NW];
    __shared__ int red_i[NW];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = warp / WPR, wi = warp % WPR;
    const int C = K >> 3;
    for (int j = threadIdx.x; j < (K >> 2); j += blockDim.x) gamma_s[j] = __ldg(reinterpret_cast<const float4*>(gamma) + j);
    __syncthreads();
    pdl_wait();  // x may come from the previous kernel (no-op unless launched as a dependent)
    pdl_launch_dependents();

    auto group_sync = [&]() {
        if constexpr (WPR > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "n"(WPR * 32) : "memory");
    };
    auto load_row = [&](int64_t m, uint4 (&v)[CH]) {
        const uint4* xr = reinterpret_cast<const uint4*>(x + m * static_cast<int64_t>(K));
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int c = wi * 32 + lane + i * (32 * WPR);
            v[i] = c < C ? __ldcs(xr + c) : make_uint4(0u, 0u, 0u, 0u);
        }
    };

    const int64_t stride = static_cast<int64_t>(gridDim.x) * RPC;
    int64_t m = static_cast<int64_t>(blockIdx.x) * RPC + grp;
    uint4 cur[CH], nxt[CH];
    if (m < M) load_row(m, cur);
    for (; m < M; m += stride) {
        if (m + stride < M) load_row(m + stride, nxt);

        // sum of squares: four fp64 chains per lane (bf16 squares are exact in fp64)
        double s2[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            float f[8];
            unpack_bf16x8(cur[i], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) s2[e & 3] += static_cast<double>(f[e]) * static_cast<double>(f[e]);
        }
        double s2w = warp_sum_f64((s2[0] + s2[1]) + (s2[2] + s2[3]));
        if constexpr (WPR > 1) {
            if (lane == 0) red_d[warp] = s2w;
            group_sync();
            s2w = red_d[grp * WPR];
#pragma unroll
            for (int i = 1; i < WPR; ++i) s2w += red_d[grp * WPR + i];
        }
        const float ms = static_cast<float>(s2w / static_cast<double>(K));
        const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));

        float amax[2] = {0.0f, 0.0f};
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int c = wi * 32 + lane + i * (32 * WPR);
            if (c < C) {
                float f[8];
                unpack_bf16x8(cur[i], f);
                const float4 ga = gamma_s[2 * c], gb = gamma_s[2 * c + 1];
                const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    amax[e & 1] = fmaxf(amax[e & 1], fabsf(__fmul_rn(__fmul_rn(f[e], inv), g[e])));
            }
        }
        // amax >= 0, so its bits order like unsigned integers
        float amax_w = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(amax[0], amax[1]))));
        if constexpr (WPR > 1) {
            if (lane == 0) red_f[warp] = amax_w;
            group_sync();
            amax_w = red_f[grp * WPR];
#pragma unroll
            for (int i = 1; i < WPR; ++i) amax_w = fmaxf(amax_w, red_f[grp * WPR + i]);
        }
        const float a = fmaxf(amax_w, 1e-5f);
        const float s = __fdiv_rn(127.0f, a);

        int qs = 0;
        uint2* qr = reinterpret_cast<uint2*>(q + m * static_cast<int64_t>(K));
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int c = wi * 32 + lane + i * (32 * WPR);
            if (c < C) {
                float f[8];
                unpack_bf16x8(cur[i], f);
                const float4 ga = gamma_s[2 * c], gb = gamma_s[2 * c + 1];
                const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                uint32_t cb[8];  // codes in the low bytes
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    cb[e] = __float_as_uint(
                        __fadd_rn(__fmul_rn(__fmul_rn(__fmul_rn(f[e], inv), g[e]), s), 12582912.0f));
                const uint32_t w0 =
                    __byte_perm(__byte_perm(cb[0], cb[1], 0x0040), __byte_perm(cb[2], cb[3], 0x0040), 0x5410);
                const uint32_t w1 =
                    __byte_perm(__byte_perm(cb[4], cb[5], 0x0040), __byte_perm(cb[6], cb[7], 0x0040), 0x5410);
                qs = __dp4a(static_cast<int>(w0), 0x01010101, qs);
                qs = __dp4a(static_cast<int>(w1), 0x01010101, qs);
                __stcs(qr + c, make_uint2(w0, w1));
            }
        }
        qs = __reduce_add_sync(0xffffffffu, qs);
        if constexpr (WPR > 1) {
            if (lane == 0) red_i[warp] = qs;
            group_sync();
            qs = red_i[grp * WPR];
#pragma unroll
            for (int i = 1; i < WPR; ++i) qs += red_i[grp * WPR + i];
        }
        if (wi == 0 && lane == 0) {
            absmax[m] = a;
            if (qsum) qsum[m] = qs;
        }
#pragma unroll
        for (int i = 0; i < CH; ++i) cur[i] = nxt[i];
    }
}

// qsum only (for the contraction alone, when q is given); with bl_nt > 0 it
// also copies the codes into the decode tensor-core kernel's operand layout (grid
// bl_nt: rows M .. bl_nt - 1 are written as zeros and get no sum).
__global__ void __launch_bounds__(kQuantThreads) qsum_kernel(const int8_t* __restrict__ q, int K, int64_t M,
                                                             int* __restrict__ qsum, int8_t* __restrict__ bl,
                                                             int bl_nt) {
    __shared__ int red_i[kQuantThreads / 32 + 1];
    const int64_t m = blockIdx.x;
    if (m >= M) {
        for (int c = threadIdx.x; c < (K >> 3); c += kQuantThreads)
            *reinterpret_cast<uint2*>(bl + blayout_offset(m, c, bl_nt)) = make_uint2(0u, 0u);
        return;  // uniform for the CTA
    }
    const uint2* qr = reinterpret_cast<const uint2*>(q + m * static_cast<int64_t>(K));
    int s = 0;
    for (int c = threadIdx.x; c < (K >> 3); c += kQuantThreads) {
        const uint2 v = __ldg(qr + c);
        s += __dp4a(static_cast<int>(v.x), 0x01010101, 0);
        s += __dp4a(static_cast<int>(v.y), 0x01010101, 0);
        if (bl_nt > 0) *reinterpret_cast<uint2*>(bl + blayout_offset(m, c, bl_nt)) = v;
    }
    s = block_allreduce(s, red_i, AddOp());
    if (threadIdx.x == 0) qsum[m] = s;
}

}  // namespace mmf
