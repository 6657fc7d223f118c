// gemv.cuh -- decode-regime fused BitLinear (small M): RMSNorm + int8
// quantisation of the M tokens into shared memory, then the ternary
// contraction over a stream of 2-bit packed weights on CUDA cores.
//
// The contraction follows the pages' ternary rule (ld246.com, section
// "三值权重的应用": +1 adds the input, -1 subtracts it, 0 skips it).  The
// packed code of a weight is c = w~ + 1 in {0, 1, 2}, so
//     sum_k w~_k q_k = sum_k c_k q_k - sum_k q_k,
// where c_k q_k adds q_k zero, one or two times.  Four codes sit in the four
// bytes of a word under one mask, each multiplied in place by a power of four
// (mask j = 0x03030303 << 2j leaves c * 4^j in every byte), so one LOP3 plus
// one DP4A adds four selected activation bytes into an int32 lane; the four
// power-of-four lanes are shifted back and summed once per row, and the
// per-token sum_k q_k is subtracted once.  All integer, exact.
//
// CTA: 8 compute warps + 1 producer warp.  The CTA owns a contiguous range of
// output rows; the producer first bulk-copies (TMA) the M rows of x into shared
// memory, then streams the CTA's weight rows (contiguous in memory) into a ring
// of shared-memory stages, so the weight fetch overlaps the normalisation.  Compute
// warps take groups of 4 rows; 8 lanes cover one row, lane l reading 16-byte
// chunks l, l+8, ... (64 weights each); a row's 8 partials meet in a 3-step
// warp-shuffle tree.
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kGemvComputeWarps = 8;
constexpr int kGemvThreads = (kGemvComputeWarps + 1) * 32;
constexpr int kGemvStages = 4;
constexpr int kGemvMaxTokens = 8;
constexpr int kGemvStageTarget = 32768;  // bytes of packed weights per stage

struct GemvParams {
    const uint16_t* x;       // bf16 [M][K]      (fused mode)
    const float* gamma;      // fp32 [K]         (fused mode)
    const int8_t* q_in;      // int8 [M][K]      (contraction-only mode)
    const uint32_t* packed;  // [N][K/16]
    const float* scale;      // beta             (fused mode)
    uint16_t* y;             // bf16 [M][N]      (fused mode)
    int32_t* acc;            // int32 [M][N]     (contraction-only mode)
    float eps;
    int M, K, N;
    int rows_per_stage;      // multiple of 4
    int rows_per_cta;
    int stage_bytes;         // rows_per_stage * K/4
    int stages;              // 2 .. kGemvStages
};

constexpr int kGemvSmemBudget = 200 * 1024;

// Host-side shape of the launch; returns false if the shape does not fit.
// Shared memory: `stages` weight stages, the M bf16 rows of x (3 bytes per
// activation with their int8 codes).  The plan depends only on (M, K, N) and
// the SM count; feasibility depends only on (M, K).
struct GemvPlan {
    int rows_per_stage, stage_bytes, rows_per_cta, grid, stages;
    size_t smem_bytes;
};

inline bool gemv_plan(int M, int K, int N, int num_sms, GemvPlan* plan) {
    if (M < 1 || M > kGemvMaxTokens) return false;
    const int rowbytes = K / 4;
    const size_t act = static_cast<size_t>(3) * M * K;
    int rs = 4 * (kGemvStageTarget / (4 * rowbytes));
    if (rs > 64) rs = 64;
    int st = kGemvStages;
    for (;;) {
        if (rs < 4) return false;
        if (static_cast<size_t>(st) * rs * rowbytes + act <= static_cast<size_t>(kGemvSmemBudget)) break;
        if (st > 2) --st;
        else rs -= 4;
    }
    plan->rows_per_stage = rs;
    plan->stage_bytes = rs * rowbytes;
    plan->stages = st;
    int grid = (N + 3) / 4;
    if (grid > num_sms) grid = num_sms;
    if (grid < 1) grid = 1;
    int per = (N + grid - 1) / grid;
    per = (per + 3) & ~3;
    plan->rows_per_cta = per;
    plan->grid = (N + per - 1) / per;
    plan->smem_bytes = static_cast<size_t>(st) * plan->stage_bytes + act;
    return true;
}

__device__ __forceinline__ void gemv_compute_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kGemvComputeWarps * 32) : "memory");
}

template <int MT, bool FUSED>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const GemvParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t full_bar[kGemvStages];
    __shared__ __align__(8) uint64_t empty_bar[kGemvStages];
    __shared__ __align__(8) uint64_t act_bar;
    __shared__ int qsum_s[MT];
    __shared__ float cm_s[MT];
    __shared__ double red_d[kGemvComputeWarps];
    __shared__ float red_f[kGemvComputeWarps];
    __shared__ int red_i[kGemvComputeWarps];
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int K = p.K;
    const int rowbytes = K >> 2;
    const int S = p.stages;
    const int row0 = blockIdx.x * p.rows_per_cta;
    const int nrows = min(p.N - row0, p.rows_per_cta);
    if (nrows <= 0) return;  // uniform for the whole CTA, before any barrier
    const int nst = (nrows + p.rows_per_stage - 1) / p.rows_per_stage;

    uint8_t* ring = smem;
    uint8_t* act = smem + static_cast<size_t>(S) * p.stage_bytes;
    const uint16_t* x_s = reinterpret_cast<const uint16_t*>(act);                 // fused: M x K bf16
    int8_t* q_s = reinterpret_cast<int8_t*>(act + (FUSED ? 2 * static_cast<size_t>(p.M) * K : 0));
    const uint32_t act_bytes = static_cast<uint32_t>((FUSED ? 2 : 1) * static_cast<size_t>(p.M) * K);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kGemvComputeWarps);
        }
        mbar_init(&act_bar, 1);
        abort_flag = 0;
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == kGemvComputeWarps) {
        // ---------------- producer: activations, then packed weight rows -> ring
        if (lane == 0) {
            mbar_arrive_expect_tx(&act_bar, act_bytes);
            if constexpr (FUSED) bulk_g2s(act, p.x, act_bytes, &act_bar);
            else bulk_g2s(q_s, p.q_in, act_bytes, &act_bar);
            const uint8_t* src = reinterpret_cast<const uint8_t*>(p.packed) + static_cast<size_t>(row0) * rowbytes;
            int issued = 0;
            for (int s = 0; s < nst; ++s) {
                const int slot = s % S;
                if (s >= S && !mbar_wait(&empty_bar[slot], ((s / S) - 1) & 1, &abort_flag)) break;
                const int r = min(p.rows_per_stage, nrows - s * p.rows_per_stage);
                const uint32_t bytes = static_cast<uint32_t>(r) * rowbytes;
                mbar_arrive_expect_tx(&full_bar[slot], bytes);
                bulk_g2s(ring + static_cast<size_t>(slot) * p.stage_bytes,
                         src + static_cast<size_t>(s) * p.rows_per_stage * rowbytes, bytes, &full_bar[slot]);
                ++issued;
            }
            // Let every copy this CTA started land before the CTA can exit.
            int zero = 0;
            mbar_wait(&act_bar, 0, &zero);
            for (int s = max(0, issued - S); s < issued; ++s) mbar_wait(&full_bar[s % S], (s / S) & 1, &zero);
        }
        return;
    }

    // ---------------- compute warps: RMSNorm + int8 quantisation of the M tokens.
    // Token m is shared by WPT = 8 / MP warps (MP = M rounded up to a power of
    // two); every reduction is per-thread sequential, a warp xor-tree, then the
    // group's warps in index order, so the result does not vary run to run.
    constexpr int MP = MT <= 1 ? 1 : (MT <= 2 ? 2 : (MT <= 4 ? 4 : 8));
    constexpr int WPT = kGemvComputeWarps / MP;
    const int m = warp / WPT;
    const bool active = m < p.M;
    const int tg = (warp % WPT) * 32 + lane;
    const int w0 = m * WPT;
    const bool act_ok = mbar_wait(&act_bar, 0, &abort_flag);
    if constexpr (FUSED) {
        const int C8 = K >> 3;
        const uint4* xr = reinterpret_cast<const uint4*>(x_s + static_cast<size_t>(m) * K);
        const float4* g4 = reinterpret_cast<const float4*>(p.gamma);
        double s2 = 0.0;
        if (active && act_ok) {
            for (int c = tg; c < C8; c += 32 * WPT) {
                const uint4 v = xr[c];
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const double lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
                    s2 += lo * lo + hi * hi;
                }
            }
        }
        s2 = warp_sum_f64(s2);
        if (lane == 0) red_d[warp] = s2;
        gemv_compute_sync();
        s2 = 0.0;
#pragma unroll
        for (int i = 0; i < WPT; ++i) s2 += red_d[(w0 + i) % kGemvComputeWarps];
        const float ms = static_cast<float>(s2 / static_cast<double>(K));
        const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, p.eps)));

        float amax = 0.0f;
        if (active && act_ok) {
            for (int c = tg; c < C8; c += 32 * WPT) {
                const uint4 v = xr[c];
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                const float4 ga = __ldg(g4 + 2 * c), gb = __ldg(g4 + 2 * c + 1);
                const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    amax = fmaxf(amax, fabsf(__fmul_rn(__fmul_rn(__uint_as_float(w[i] << 16), inv), g[2 * i])));
                    amax = fmaxf(amax,
                                 fabsf(__fmul_rn(__fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv), g[2 * i + 1])));
                }
            }
        }
        amax = warp_max_f32(amax);
        if (lane == 0) red_f[warp] = amax;
        gemv_compute_sync();
        amax = 0.0f;
#pragma unroll
        for (int i = 0; i < WPT; ++i) amax = fmaxf(amax, red_f[(w0 + i) % kGemvComputeWarps]);
        const float a = fmaxf(amax, 1e-5f);
        const float s = __fdiv_rn(127.0f, a);

        int qs = 0;
        if (active && act_ok) {
            uint2* qrow = reinterpret_cast<uint2*>(q_s + static_cast<size_t>(m) * K);
            for (int c = tg; c < C8; c += 32 * WPT) {
                const uint4 v = xr[c];
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                const float4 ga = __ldg(g4 + 2 * c), gb = __ldg(g4 + 2 * c + 1);
                const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                uint32_t out[2] = {0u, 0u};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float xv =
                        (i & 1) ? __uint_as_float(w[i >> 1] & 0xFFFF0000u) : __uint_as_float(w[i >> 1] << 16);
                    const int code = quant_code(__fmul_rn(__fmul_rn(xv, inv), g[i]), s);
                    qs += code;
                    out[i >> 2] |= (static_cast<uint32_t>(code) & 0xFFu) << (8 * (i & 3));
                }
                qrow[c] = make_uint2(out[0], out[1]);
            }
        }
        qs = warp_sum_i32(qs);
        if (lane == 0) red_i[warp] = qs;
        gemv_compute_sync();
        if (active && tg == 0) {
            int t = 0;
#pragma unroll
            for (int i = 0; i < WPT; ++i) t += red_i[w0 + i];
            qsum_s[m] = t;
            cm_s[m] = __fmul_rn(__fdiv_rn(a, 127.0f), __ldg(p.scale));
        }
    } else {
        int qs = 0;
        if (active && act_ok) {
            const uint4* qr = reinterpret_cast<const uint4*>(q_s + static_cast<size_t>(m) * K);
            for (int c = tg; c < (K >> 4); c += 32 * WPT) {
                const uint4 v = qr[c];
                qs = __dp4a(static_cast<int>(v.x), 0x01010101, qs);
                qs = __dp4a(static_cast<int>(v.y), 0x01010101, qs);
                qs = __dp4a(static_cast<int>(v.z), 0x01010101, qs);
                qs = __dp4a(static_cast<int>(v.w), 0x01010101, qs);
            }
        }
        qs = warp_sum_i32(qs);
        if (lane == 0) red_i[warp] = qs;
        gemv_compute_sync();
        if (active && tg == 0) {
            int t = 0;
#pragma unroll
            for (int i = 0; i < WPT; ++i) t += red_i[w0 + i];
            qsum_s[m] = t;
        }
    }
    gemv_compute_sync();
    if (!act_ok) return;

    // ---------------- contraction over the staged rows
    const int g_row = lane >> 3;  // row within a group of 4
    const int l8 = lane & 7;      // lane within the row
    const int C = K >> 6;         // 16-byte chunks (64 weights) per row
    for (int s = 0; s < nst; ++s) {
        const int slot = s % S;
        const bool ok = mbar_wait(&full_bar[slot], (s / S) & 1, &abort_flag);
        if (!ok) break;
        const int rs = min(p.rows_per_stage, nrows - s * p.rows_per_stage);
        const int ngroups = (rs + 3) >> 2;
        const uint8_t* stage = ring + static_cast<size_t>(slot) * p.stage_bytes;
        for (int grp = warp; grp < ngroups; grp += kGemvComputeWarps) {
            const int rl = 4 * grp + g_row;
            const bool valid = rl < rs;
            int acc[MT][4];
#pragma unroll
            for (int mm = 0; mm < MT; ++mm)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[mm][j] = 0;
            if (valid) {
                const uint4* wrow = reinterpret_cast<const uint4*>(stage + static_cast<size_t>(rl) * rowbytes);
#pragma unroll 2
                for (int c = l8; c < C; c += 8) {
                    const uint4 wv = wrow[c];
                    const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const uint32_t m0 = wd[t] & 0x03030303u, m1 = wd[t] & 0x0C0C0C0Cu;
                        const uint32_t m2 = wd[t] & 0x30303030u, m3 = wd[t] & 0xC0C0C0C0u;
#pragma unroll
                        for (int mm = 0; mm < MT; ++mm) {
                            const uint4 qv =
                                *reinterpret_cast<const uint4*>(q_s + static_cast<size_t>(mm) * K + 64 * c + 16 * t);
                            acc[mm][0] = dp4a_us(m0, qv.x, acc[mm][0]);
                            acc[mm][1] = dp4a_us(m1, qv.y, acc[mm][1]);
                            acc[mm][2] = dp4a_us(m2, qv.z, acc[mm][2]);
                            acc[mm][3] = dp4a_us(m3, qv.w, acc[mm][3]);
                        }
                    }
                }
            }
            const int n = row0 + s * p.rows_per_stage + rl;
#pragma unroll
            for (int mm = 0; mm < MT; ++mm) {
                int t = acc[mm][0] + (acc[mm][1] >> 2) + (acc[mm][2] >> 4) + (acc[mm][3] >> 6);
                t += __shfl_xor_sync(0xffffffffu, t, 1);
                t += __shfl_xor_sync(0xffffffffu, t, 2);
                t += __shfl_xor_sync(0xffffffffu, t, 4);
                if (valid && l8 == 0 && mm < p.M) {
                    const int v = t - qsum_s[mm];
                    if constexpr (FUSED) {
                        const __nv_bfloat16 yb = __float2bfloat16_rn(__fmul_rn(static_cast<float>(v), cm_s[mm]));
                        p.y[static_cast<size_t>(mm) * p.N + n] = __bfloat16_as_ushort(yb);
                    } else {
                        p.acc[static_cast<size_t>(mm) * p.N + n] = v;
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[slot]);
    }
}

}  // namespace mmf
