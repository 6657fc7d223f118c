// gemv.cuh -- decode-regime fused BitLinear (small M): RMSNorm + int8
// quantisation of the M tokens in shared memory, then the ternary contraction
// over a stream of 2-bit packed weights on CUDA cores.  One launch serves a
// group of up to kGemvMaxProj projections that share the input x (the token
// mixer's gate projections, the channel mixer's gate/up pair).
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
// CTA: 8 compute warps + 1 producer warp.  The group's weight rows form one
// concatenated row space; each CTA owns a contiguous range of it.  The
// producer bulk-copies (TMA) the CTA's weight rows into a ring of small
// shared-memory stages and gamma into shared memory, then waits for the
// previous kernel on the stream (programmatic dependent launch; a no-op when
// the launch is not programmatic), then copies the M rows of x.  So under PDL
// the weight stream overlaps the previous kernel and only x waits for it.
// Compute warps take groups of 4 rows; 8 lanes cover one row, lane l reading
// 16-byte chunks l, l+8, ... (64 weights each); a row's 8 partials meet in a
// 3-step warp-shuffle tree.
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kGemvComputeWarps = 8;
constexpr int kGemvThreads = (kGemvComputeWarps + 1) * 32;
constexpr int kGemvMaxStages = 8;
constexpr int kGemvMaxTokens = 8;
constexpr int kGemvMaxProj = 8;
constexpr int kGemvStageTarget = 8192;       // bytes of packed weights per stage
constexpr int kGemvSmemTwoCta = 110 * 1024;  // two CTAs per SM fit under this
constexpr int kGemvSmemBudget = 200 * 1024;

struct GemvParams {
    const uint16_t* x;                      // bf16 [M][K]      (fused mode)
    const float* gamma;                     // fp32 [K]         (fused mode)
    const int8_t* q_in;                     // int8 [M][K]      (contraction-only mode)
    const uint32_t* packed[kGemvMaxProj];   // [N_g][K/16]
    const float* scale[kGemvMaxProj];       // beta_g           (fused mode)
    uint16_t* y[kGemvMaxProj];              // bf16 [M][N_g]    (fused mode)
    int32_t* acc;                           // int32 [M][N]     (contraction-only mode, one projection)
    int row_start[kGemvMaxProj + 1];        // prefix sums of N_g
    float eps;
    int M, K, nproj;
    int rows_per_stage;                     // multiple of 4
    int rows_per_cta;
    int stage_bytes;                        // rows_per_stage * K/4
    int stages;                             // 1 .. kGemvMaxStages
};

// Host-side shape of the launch; returns false if the shape does not fit.
// Shared memory holds `stages` weight stages and the activations: x (bf16),
// its int8 codes and gamma (fp32).  Feasibility depends only on (M, K).
struct GemvPlan {
    int rows_per_stage, stage_bytes, rows_per_cta, grid, stages;
    size_t smem_bytes;
};

inline size_t gemv_act_bytes(int M, int K) { return static_cast<size_t>(3) * M * K + static_cast<size_t>(4) * K; }

inline bool gemv_plan(int M, int K, int64_t R, int num_sms, GemvPlan* plan) {
    if (M < 1 || M > kGemvMaxTokens || R < 1) return false;
    const int rowbytes = K / 4;
    const size_t act = gemv_act_bytes(M, K);
    int rs = 4 * (kGemvStageTarget / (4 * rowbytes));
    if (rs < 4) rs = 4;
    if (rs > 64) rs = 64;
    int grid = static_cast<int>((R + 3) / 4);
    if (grid > num_sms) grid = num_sms;
    int per = static_cast<int>((R + grid - 1) / grid);
    per = (per + 3) & ~3;
    const int want = (per + rs - 1) / rs;  // stages that hold the CTA's whole slab
    // Prefer a ring that holds the whole slab within the two-CTA budget, then
    // fewer stages, then the one-CTA budget, then smaller stages.
    const size_t budgets[2] = {static_cast<size_t>(kGemvSmemTwoCta), static_cast<size_t>(kGemvSmemBudget)};
    for (size_t budget : budgets) {
        for (int r = rs; r >= 4; r -= 4) {
            int st = want < kGemvMaxStages ? want : kGemvMaxStages;
            if (r != rs) st = (per + r - 1) / r < kGemvMaxStages ? (per + r - 1) / r : kGemvMaxStages;
            for (; st >= 1; --st) {
                if (static_cast<size_t>(st) * r * rowbytes + act <= budget) {
                    if (st < 2 && budget == budgets[0]) break;  // two-CTA plans keep a double buffer
                    plan->rows_per_stage = r;
                    plan->stage_bytes = r * rowbytes;
                    plan->stages = st;
                    plan->rows_per_cta = per;
                    plan->grid = static_cast<int>((R + per - 1) / per);
                    plan->smem_bytes = static_cast<size_t>(st) * plan->stage_bytes + act;
                    return true;
                }
            }
        }
    }
    return false;
}

__device__ __forceinline__ void gemv_compute_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kGemvComputeWarps * 32) : "memory");
}

// projection of a global row (row_start is short and sorted)
__device__ __forceinline__ int gemv_proj_of(const GemvParams& p, int r) {
    int g = 0;
#pragma unroll
    for (int i = 1; i < kGemvMaxProj; ++i)
        if (i < p.nproj && r >= p.row_start[i]) g = i;
    return g;
}

template <int MT, bool FUSED>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const __grid_constant__ GemvParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t full_bar[kGemvMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kGemvMaxStages];
    __shared__ __align__(8) uint64_t act_bar;
    __shared__ int qsum_s[MT];
    __shared__ float deq_s[MT];
    __shared__ float beta_s[kGemvMaxProj];
    __shared__ double red_d[kGemvComputeWarps];
    __shared__ float red_f[kGemvComputeWarps];
    __shared__ int red_i[kGemvComputeWarps];
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int K = p.K;
    const int rowbytes = K >> 2;
    const int S = p.stages;
    const int R = p.row_start[p.nproj];
    const int row0 = blockIdx.x * p.rows_per_cta;
    const int nrows = min(R - row0, p.rows_per_cta);
    if (nrows <= 0) return;  // uniform for the whole CTA, before any barrier
    const int nst = (nrows + p.rows_per_stage - 1) / p.rows_per_stage;

    // shared memory: [ring: S stages][gamma fp32 K][x bf16 M*K][q int8 M*K]
    uint8_t* ring = smem;
    float* gamma_s = reinterpret_cast<float*>(smem + static_cast<size_t>(S) * p.stage_bytes);
    uint16_t* x_s = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(gamma_s) + 4 * static_cast<size_t>(K));
    int8_t* q_s = reinterpret_cast<int8_t*>(reinterpret_cast<uint8_t*>(x_s) + 2 * static_cast<size_t>(p.M) * K);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kGemvComputeWarps);
        }
        mbar_init(&act_bar, 1);
        abort_flag = 0;
        mbar_fence_init();
    }
    if (FUSED && threadIdx.x < p.nproj) beta_s[threadIdx.x] = __ldg(p.scale[threadIdx.x]);
    __syncthreads();

    if (warp == kGemvComputeWarps) {
        // ---------------- producer
        if (lane == 0) {
            auto issue_stage = [&](int s) {
                const int slot = s % S;
                const int r0 = row0 + s * p.rows_per_stage;
                const int r1 = r0 + min(p.rows_per_stage, nrows - s * p.rows_per_stage);
                mbar_arrive_expect_tx(&full_bar[slot], static_cast<uint32_t>(r1 - r0) * rowbytes);
                uint8_t* dst = ring + static_cast<size_t>(slot) * p.stage_bytes;
                for (int r = r0; r < r1;) {  // split at projection boundaries
                    const int g = gemv_proj_of(p, r);
                    const int e = min(r1, p.row_start[g + 1]);
                    const uint8_t* src = reinterpret_cast<const uint8_t*>(p.packed[g]) +
                                         static_cast<size_t>(r - p.row_start[g]) * rowbytes;
                    bulk_g2s(dst + static_cast<size_t>(r - r0) * rowbytes, src,
                             static_cast<uint32_t>(e - r) * rowbytes, &full_bar[slot]);
                    r = e;
                }
            };
            // weights and gamma are parameters: fetched before the dependency wait
            const int first = min(nst, S);
            for (int s = 0; s < first; ++s) issue_stage(s);
            const uint32_t x_bytes = static_cast<uint32_t>((FUSED ? 2 : 1) * static_cast<size_t>(p.M) * K);
            const uint32_t g_bytes = FUSED ? 4u * static_cast<uint32_t>(K) : 0u;
            mbar_arrive_expect_tx(&act_bar, x_bytes + g_bytes);
            if constexpr (FUSED) bulk_g2s(gamma_s, p.gamma, g_bytes, &act_bar);
            // activations may come from the previous kernel on the stream
            pdl_wait();
            if constexpr (FUSED) bulk_g2s(x_s, p.x, x_bytes, &act_bar);
            else bulk_g2s(q_s, p.q_in, x_bytes, &act_bar);
            pdl_launch_dependents();
            int issued = first;
            for (int s = first; s < nst; ++s) {
                if (!mbar_wait(&empty_bar[s % S], ((s / S) - 1) & 1, &abort_flag)) break;
                issue_stage(s);
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
        const float4* g4 = reinterpret_cast<const float4*>(gamma_s);
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
                const float4 ga = g4[2 * c], gb = g4[2 * c + 1];
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
                const float4 ga = g4[2 * c], gb = g4[2 * c + 1];
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
            deq_s[m] = __fdiv_rn(a, 127.0f);
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
            const int r = row0 + s * p.rows_per_stage + rl;
            const int g = gemv_proj_of(p, valid ? r : row0);
            const int n = r - p.row_start[g];
            const int Ng = p.row_start[g + 1] - p.row_start[g];
#pragma unroll
            for (int mm = 0; mm < MT; ++mm) {
                int t = acc[mm][0] + (acc[mm][1] >> 2) + (acc[mm][2] >> 4) + (acc[mm][3] >> 6);
                t += __shfl_xor_sync(0xffffffffu, t, 1);
                t += __shfl_xor_sync(0xffffffffu, t, 2);
                t += __shfl_xor_sync(0xffffffffu, t, 4);
                if (valid && l8 == 0 && mm < p.M) {
                    const int v = t - qsum_s[mm];
                    if constexpr (FUSED) {
                        const float cm = __fmul_rn(deq_s[mm], beta_s[g]);
                        const __nv_bfloat16 yb = __float2bfloat16_rn(__fmul_rn(static_cast<float>(v), cm));
                        p.y[g][static_cast<size_t>(mm) * Ng + n] = __bfloat16_as_ushort(yb);
                    } else {
                        p.acc[static_cast<size_t>(mm) * Ng + n] = v;
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[slot]);
    }
}

}  // namespace mmf
