// scan.cuh -- the MLGRU token mixer's element-wise recurrence, the part of the
// token mixer between its f/c/g projections and its o projection
// (datacamp.com, section "Các thành phần lõi: MLGRU và GLU": tokens one at a
// time, gates in (0, 1) mixing the previous hidden state and the current
// token).  Per sequence b and channel k, token by token:
//   f = sigma(f_pre), c = SiLU(c_pre), g = sigma(g_pre)
//   h = f * h + (1 - f) * c           (fp32 state)
//   o = bf16(g * h)                   (the o projection's input)
//
// The recurrence is linear in h, h_t = f_t h_{t-1} + (1 - f_t) c_t, so a chunk
// of tokens acts on its incoming state as h -> A h + B with A the product of
// its f and B its result from h = 0.  A CTA takes 64 channels of one sequence
// (lane = a channel pair, bf16x2 loads) and splits the tokens into one chunk
// per warp: pass 1 forms each chunk's (A, B), the warps combine the chunks
// before theirs in order to get their incoming state, and pass 2 runs the
// recurrence over the chunk from it and writes o.  HBM: the pre-activations
// are read twice (the second time mostly from L2) and o written once.
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kScanWarps = 32;

// sigma(v) = 1 / (1 + e^-v) with the hardware exponential and reciprocal
// (a few ulp: the recurrence is bound by the transcendental pipe with the
// IEEE forms, and its state is compared with the oracle to fp32-level
// tolerances anyway).  The sigmoids of one token share one reciprocal:
// with d_i = 1 + e^-v_i, 1 / (d_1 d_2) gives sigma(v_1) = d_2 / (d_1 d_2)
// and sigma(v_2) = d_1 / (d_1 d_2) (three of the pipe's operations instead of
// four; five instead of six for three sigmoids).  Inputs are clamped below at
// -28 so that a product of three d stays finite (e^28 < 1.5e12); sigma(-28)
// is 7e-13, so the clamp changes a gate by less than that.
constexpr float kScanClamp = -28.0f;

__device__ __forceinline__ float sig_den(float v) { return 1.0f + __expf(-fmaxf(v, kScanClamp)); }

__device__ __forceinline__ void sigmoid2(float a, float b, float& sa, float& sb) {
    const float da = sig_den(a), db = sig_den(b);
    const float r = __fdividef(1.0f, da * db);
    sa = r * db;
    sb = r * da;
}

__device__ __forceinline__ void sigmoid3(float a, float b, float c, float& sa, float& sb, float& sc) {
    const float da = sig_den(a), db = sig_den(b), dc = sig_den(c);
    const float dab = da * db;
    const float r = __fdividef(1.0f, dab * dc);
    const float rc = r * dc;  // 1 / (da db)
    sa = rc * db;
    sb = rc * da;
    sc = r * dab;
}

__device__ __forceinline__ void bf16x2_to_f(uint32_t w, float& lo, float& hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
}

__global__ void __launch_bounds__(kScanWarps * 32, 1) mlgru_scan_kernel(const uint16_t* __restrict__ f_pre,
                                                                     const uint16_t* __restrict__ c_pre,
                                                                     const uint16_t* __restrict__ g_pre,
                                                                     const float* __restrict__ h0, int T, int D,
                                                                     uint16_t* __restrict__ o,
                                                                     float* __restrict__ h_last) {
    __shared__ float2 agg_a[kScanWarps][32];
    __shared__ float2 agg_b[kScanWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t b = blockIdx.y;
    const int k = blockIdx.x * 64 + 2 * lane;  // this lane's channels k, k + 1
    const bool valid = k < D;                  // D is even, so k + 1 < D too
    const int L = (T + kScanWarps - 1) / kScanWarps;
    const int t0 = min(T, warp * L), t1 = min(T, t0 + L);
    auto idx = [&](int t) { return (b * T + t) * static_cast<int64_t>(D) + k; };

    // pass 1: the chunk's map h -> A h + B
    float a0 = 1.0f, a1 = 1.0f, b0 = 0.0f, b1 = 0.0f;
    if (valid) {
#pragma unroll 8
        for (int t = t0; t < t1; ++t) {
            float fp0, fp1, cp0, cp1;
            bf16x2_to_f(__ldg(reinterpret_cast<const uint32_t*>(f_pre + idx(t))), fp0, fp1);
            bf16x2_to_f(__ldg(reinterpret_cast<const uint32_t*>(c_pre + idx(t))), cp0, cp1);
            float f0, f1, sc0, sc1;
            sigmoid2(fp0, cp0, f0, sc0);
            sigmoid2(fp1, cp1, f1, sc1);
            const float c0 = __fmul_rn(cp0, sc0), c1 = __fmul_rn(cp1, sc1);
            b0 = __fadd_rn(__fmul_rn(f0, b0), __fmul_rn(__fsub_rn(1.0f, f0), c0));
            b1 = __fadd_rn(__fmul_rn(f1, b1), __fmul_rn(__fsub_rn(1.0f, f1), c1));
            a0 = __fmul_rn(a0, f0);
            a1 = __fmul_rn(a1, f1);
        }
    }
    agg_a[warp][lane] = make_float2(a0, a1);
    agg_b[warp][lane] = make_float2(b0, b1);
    __syncthreads();

    // incoming state: h0 through the chunks before this one, in order
    float h0v = 0.0f, h1v = 0.0f;
    if (valid && h0) {
        const float2 hv = *reinterpret_cast<const float2*>(h0 + b * D + k);
        h0v = hv.x;
        h1v = hv.y;
    }
    for (int w = 0; w < warp; ++w) {
        const float2 aw = agg_a[w][lane], bw = agg_b[w][lane];
        h0v = __fadd_rn(__fmul_rn(aw.x, h0v), bw.x);
        h1v = __fadd_rn(__fmul_rn(aw.y, h1v), bw.y);
    }

    // pass 2: the recurrence over the chunk, writing o
    if (valid) {
#pragma unroll 8
        for (int t = t0; t < t1; ++t) {
            float fp0, fp1, cp0, cp1, gp0, gp1;
            bf16x2_to_f(__ldg(reinterpret_cast<const uint32_t*>(f_pre + idx(t))), fp0, fp1);
            bf16x2_to_f(__ldg(reinterpret_cast<const uint32_t*>(c_pre + idx(t))), cp0, cp1);
            bf16x2_to_f(__ldg(reinterpret_cast<const uint32_t*>(g_pre + idx(t))), gp0, gp1);
            float f0, f1, sc0, sc1, g0, g1;
            sigmoid3(fp0, cp0, gp0, f0, sc0, g0);
            sigmoid3(fp1, cp1, gp1, f1, sc1, g1);
            const float c0 = __fmul_rn(cp0, sc0), c1 = __fmul_rn(cp1, sc1);
            h0v = __fadd_rn(__fmul_rn(f0, h0v), __fmul_rn(__fsub_rn(1.0f, f0), c0));
            h1v = __fadd_rn(__fmul_rn(f1, h1v), __fmul_rn(__fsub_rn(1.0f, f1), c1));
            const __nv_bfloat162 ov = __floats2bfloat162_rn(__fmul_rn(g0, h0v), __fmul_rn(g1, h1v));
            *reinterpret_cast<__nv_bfloat162*>(o + idx(t)) = ov;
        }
        // the state after the last token: the warp whose chunk ends at T (warp 0 when T == 0)
        if (h_last && t1 == T && (t0 < t1 || warp == 0))
            *reinterpret_cast<float2*>(h_last + b * D + k) = make_float2(h0v, h1v);
    }
}

}  // namespace mmf
