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
//
// mlgru_scan_tma_kernel is the same recurrence with each pre-activation read
// once and each gate computed once: a producer warp streams tiles of 128
// tokens x 64 channels of f, c and g into a ring of shared-memory stages by
// tensor copies; each of 16 compute warps takes 8 consecutive tokens of a
// stage, computes their gates into registers and releases the stage, forms
// its 8-token map, and after one barrier folds the maps of the warps before
// it, in order, from the state entering the stage: its own incoming state.
// The last warp also applies its own map and leaves the result, the state
// entering the next stage, in shared memory for every warp to read after the
// next stage's barrier.  Each warp runs its 8 tokens from its incoming state
// and writes o.  Needs D % 8 == 0 (16-byte row pitch for the
// tensor maps) and B * T < 2^31 rows; other shapes take mlgru_scan_kernel.
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kScanWarps = 32;

// sigma(v) = 1 / (1 + e^-v) with the hardware exponential and reciprocal
// (a few ulp: the IEEE forms cost several times the instructions, and the
// state is compared with the oracle to fp32-level tolerances anyway).  The sigmoids of one token share one reciprocal:
// with d_i = 1 + e^-v_i, 1 / (d_1 d_2) gives sigma(v_1) = d_2 / (d_1 d_2)
// and sigma(v_2) = d_1 / (d_1 d_2) (three of the pipe's operations instead of
// four; five instead of six for three sigmoids).  Inputs are clamped below at
// -28 so that a product of three d stays finite (e^28 < 1.5e12); sigma(-28)
// is 7e-13, so the clamp changes a gate by less than that.
constexpr float kScanClamp = -28.0f;

// 2^v and 1/v on the special-function unit, subnormal results flushed to
// zero.  Neither matters here: e^-v below the smallest normal float only
// occurs for v > 87, where 1 + e^-v is 1 in fp32 either way, and the clamp
// keeps the reciprocal's input below 4e36, so its result stays normal.
__device__ __forceinline__ float ex2_ftz(float v) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ float rcp_ftz(float v) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

constexpr float kLog2e = 1.4426950408889634f;   // 1 / ln 2: e^u = 2^(u / ln 2)

__device__ __forceinline__ float sig_den(float v) { return 1.0f + ex2_ftz(-kLog2e * fmaxf(v, kScanClamp)); }

__device__ __forceinline__ void sigmoid2(float a, float b, float& sa, float& sb) {
    const float da = sig_den(a), db = sig_den(b);
    const float r = rcp_ftz(da * db);
    sa = r * db;
    sb = r * da;
}

__device__ __forceinline__ void sigmoid3(float a, float b, float c, float& sa, float& sb, float& sc) {
    const float da = sig_den(a), db = sig_den(b), dc = sig_den(c);
    const float dab = da * db;
    const float r = rcp_ftz(dab * dc);
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

constexpr int kStWarps = 16;                        // compute warps
constexpr int kStTok = 8;                           // tokens per compute warp per stage
constexpr int kStRows = kStWarps * kStTok;          // tokens per stage
constexpr int kStCh = 64;                           // channels per CTA (a bf16 pair per lane)
constexpr int kStStages = 4;
constexpr uint32_t kStTileBytes = kStRows * kStCh * 2;   // one tensor's tile: 16 KB
constexpr uint32_t kStStageBytes = 3 * kStTileBytes;     // f, c, g
constexpr int kStThreads = (kStWarps + 1) * 32;          // + the producer warp
constexpr size_t kStSmemBytes = size_t(kStStages) * kStStageBytes + 2 * kStWarps * 32 * sizeof(float4) +
                                2 * kStStages * sizeof(uint64_t) + 16;

// f, c, g are [B * T rows][D] bf16 tensor maps, box 64 channels x 128 rows,
// no swizzle: row r of a tile is 128 contiguous bytes, lane l reads bytes
// 4l .. 4l + 3 of it (one wavefront per warp).  A stage of sequence b starts
// at row b * T + 128 s; rows past the sequence's end (the next sequence's, or
// zeros past the tensor) are read but given the identity map and not written.
__global__ void __launch_bounds__(kStThreads, 1) mlgru_scan_tma_kernel(const __grid_constant__ CUtensorMap mf,
                                                                      const __grid_constant__ CUtensorMap mc,
                                                                      const __grid_constant__ CUtensorMap mg,
                                                                      const float* __restrict__ h0, int T, int D,
                                                                      uint16_t* __restrict__ o,
                                                                      float* __restrict__ h_last) {
    extern __shared__ __align__(128) uint8_t smem[];   // tensor-copy destinations need 16 bytes
    uint8_t* tiles = smem;                                                       // [stage][f|c|g][row][64]
    float4* agg = reinterpret_cast<float4*>(smem + size_t(kStStages) * kStStageBytes);  // [2][warp][lane]
    uint64_t* full = reinterpret_cast<uint64_t*>(agg + 2 * kStWarps * 32);
    uint64_t* empty = full + kStStages;
    __shared__ int abort_flag;
    __shared__ float2 carry_sm[2][32];  // the state entering a stage, by stage parity (the last warp's)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y;
    const int k = blockIdx.x * kStCh + 2 * lane;   // this lane's channels k, k + 1
    const bool valid = k < D;                      // D % 8 == 0, so k + 1 < D too
    const int stages = (T + kStRows - 1) / kStRows;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int i = 0; i < kStStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kStWarps);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == kStWarps) {
        // producer: one elected lane issues the stages' three tensor copies
        if (lane == 0) {
            prefetch_tensormap(&mf);
            prefetch_tensormap(&mc);
            prefetch_tensormap(&mg);
            const int x = blockIdx.x * kStCh;
            int issued = 0;
            for (int s = 0; s < stages; ++s) {
                const int slot = s % kStStages;
                if (s >= kStStages && !mbar_wait(&empty[slot], ((s / kStStages) - 1) & 1, &abort_flag)) break;
                uint8_t* dst = tiles + size_t(slot) * kStStageBytes;
                const int y = b * T + s * kStRows;
                mbar_arrive_expect_tx(&full[slot], kStStageBytes);
                tma_load_2d(dst, &mf, x, y, &full[slot]);
                tma_load_2d(dst + kStTileBytes, &mc, x, y, &full[slot]);
                tma_load_2d(dst + 2 * kStTileBytes, &mg, x, y, &full[slot]);
                issued = s + 1;
            }
            // copies still in flight land before the CTA leaves (bounded, even after an abort)
            for (int s = issued > kStStages ? issued - kStStages : 0; s < issued; ++s) {
                const int slot = s % kStStages;
                const unsigned long long t0 = globaltimer_ns();
                while (!mbar_try_wait(&full[slot], (s / kStStages) & 1)) {
                    if (globaltimer_ns() - t0 > kWaitLimitNs) {
                        atomicOr(&g_error_word, kErrTimeout);
                        break;
                    }
                }
            }
        }
        return;
    }

    // the state entering the current stage (the same in every warp)
    float carry0 = 0.0f, carry1 = 0.0f;
    if (valid && h0) {
        const float2 hv = *reinterpret_cast<const float2*>(h0 + static_cast<int64_t>(b) * D + k);
        carry0 = hv.x;
        carry1 = hv.y;
    }
    for (int s = 0; s < stages; ++s) {
        const int slot = s % kStStages;
        const bool ok = mbar_wait(&full[slot], (s / kStStages) & 1, &abort_flag);
        float f[kStTok][2], bb[kStTok][2], g[kStTok][2];
        const int tw = s * kStRows + warp * kStTok;   // this warp's first token
        if (ok) {
            const uint8_t* st = tiles + size_t(slot) * kStStageBytes + size_t(warp * kStTok) * (kStCh * 2) + 4 * lane;
            uint32_t rf[kStTok], rc[kStTok], rg[kStTok];
#pragma unroll
            for (int i = 0; i < kStTok; ++i) {
                rf[i] = *reinterpret_cast<const uint32_t*>(st + i * (kStCh * 2));
                rc[i] = *reinterpret_cast<const uint32_t*>(st + kStTileBytes + i * (kStCh * 2));
                rg[i] = *reinterpret_cast<const uint32_t*>(st + 2 * kStTileBytes + i * (kStCh * 2));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);   // the tile is in registers: the slot may refill
#pragma unroll
            for (int i = 0; i < kStTok; ++i) {
                float fp0, fp1, cp0, cp1, gp0, gp1;
                bf16x2_to_f(rf[i], fp0, fp1);
                bf16x2_to_f(rc[i], cp0, cp1);
                bf16x2_to_f(rg[i], gp0, gp1);
                float sc0, sc1;
                sigmoid3(fp0, cp0, gp0, f[i][0], sc0, g[i][0]);
                sigmoid3(fp1, cp1, gp1, f[i][1], sc1, g[i][1]);
                bb[i][0] = __fmul_rn(__fsub_rn(1.0f, f[i][0]), __fmul_rn(cp0, sc0));
                bb[i][1] = __fmul_rn(__fsub_rn(1.0f, f[i][1]), __fmul_rn(cp1, sc1));
            }
            if (tw + kStTok > T) {   // tokens past the sequence (its last stage only): identity map
#pragma unroll
                for (int i = 0; i < kStTok; ++i)
                    if (tw + i >= T) {
                        f[i][0] = f[i][1] = 1.0f;
                        bb[i][0] = bb[i][1] = 0.0f;
                    }
            }
            // this warp's 8-token map h -> A h + B
            float a0 = 1.0f, a1 = 1.0f, m0 = 0.0f, m1 = 0.0f;
#pragma unroll
            for (int i = 0; i < kStTok; ++i) {
                m0 = __fmaf_rn(f[i][0], m0, bb[i][0]);
                m1 = __fmaf_rn(f[i][1], m1, bb[i][1]);
                a0 = __fmul_rn(a0, f[i][0]);
                a1 = __fmul_rn(a1, f[i][1]);
            }
            agg[(s & 1) * kStWarps * 32 + warp * 32 + lane] = make_float4(a0, a1, m0, m1);
        }
        // every compute warp leaves together if any wait gave up
        if (!named_barrier_and<1, kStWarps * 32>(ok)) return;

        // the state entering this stage: the last warp left it for stage s > 0
        // (the barrier above orders its store before these loads)
        if (s > 0) {
            const float2 cv = carry_sm[s & 1][lane];
            carry0 = cv.x;
            carry1 = cv.y;
        }
        // fold the maps of the warps before this one, in order: this warp's
        // incoming state; the last warp also applies its own map, which gives
        // the state entering the next stage
        float h0v = carry0, h1v = carry1;
        const float4* ag = agg + (s & 1) * kStWarps * 32 + lane;
#pragma unroll 4
        for (int w = 0; w < warp; ++w) {
            const float4 m = ag[w * 32];
            h0v = __fmaf_rn(m.x, h0v, m.z);
            h1v = __fmaf_rn(m.y, h1v, m.w);
        }
        if (warp == kStWarps - 1) {
            const float4 m = ag[warp * 32];
            carry0 = __fmaf_rn(m.x, h0v, m.z);
            carry1 = __fmaf_rn(m.y, h1v, m.w);
            carry_sm[(s + 1) & 1][lane] = make_float2(carry0, carry1);
        }
        // the 8 tokens from the incoming state
        if (valid) {
            uint16_t* orow = o + (static_cast<int64_t>(b) * T + tw) * D + k;
#pragma unroll
            for (int i = 0; i < kStTok; ++i) {
                h0v = __fmaf_rn(f[i][0], h0v, bb[i][0]);
                h1v = __fmaf_rn(f[i][1], h1v, bb[i][1]);
                if (tw + i < T)
                    *reinterpret_cast<__nv_bfloat162*>(orow + static_cast<int64_t>(i) * D) =
                        __floats2bfloat162_rn(__fmul_rn(g[i][0], h0v), __fmul_rn(g[i][1], h1v));
            }
        }
    }
    if (h_last && valid && warp == kStWarps - 1)  // the state after the last stage
        *reinterpret_cast<float2*>(h_last + static_cast<int64_t>(b) * D + k) = make_float2(carry0, carry1);
}

}  // namespace mmf
