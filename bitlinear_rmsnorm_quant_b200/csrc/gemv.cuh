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
// Compute warps take blocks of 8 rows, round-robin over the whole slab (so
// every warp works whatever the stage size); lane (r, l) of a warp covers rows
// r and r+4 of the block, reading their 16-byte chunks l, l+8, ... (64 weights
// each) against one shared load of the activation codes; a row's 8 partials
// meet in a 3-step warp-shuffle tree.
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kGemvMaxComputeWarps = 16;

// 8 compute warps + 1 producer warp.  Up to 4 tokens the registers of two
// CTAs fit in one SM, so under programmatic dependent launch a CTA of the
// next kernel can sit beside a running one and stream its weights into shared
// memory while the running one computes; beyond 4 tokens the accumulators
// take the register file and one CTA fits.
__host__ __device__ constexpr int gemv_compute_warps(int) { return 8; }
__host__ __device__ constexpr int gemv_threads(int M) { return (gemv_compute_warps(M) + 1) * 32; }
__host__ __device__ constexpr int gemv_ctas_per_sm(int M) { return M <= 4 ? 2 : 1; }
constexpr int kGemvMaxStages = 8;
constexpr int kGemvMaxTokens = 3;  // from 4 tokens the decode tensor-core kernel is faster
constexpr int kGemvMaxProj = 8;
constexpr int kGemvStageTarget = 10240;      // bytes of packed weights per stage
constexpr int kGemvBlockRows = 8;            // rows per warp work item
constexpr int kGemvSmemTwoCta = 110 * 1024;  // two CTAs per SM fit under this
constexpr int kGemvSmemBudget = 220 * 1024;   // under the 227 KB per-CTA limit with the static part

struct GemvParams {
    const uint16_t* x;                      // bf16 [M][K]      (fused mode; the gate g in GLU mode)
    const uint16_t* u;                      // bf16 [M][K]      (GLU mode: p = bf16(SiLU(g) * u) is normalised)
    const float* gamma;                     // fp32 [K]         (fused mode)
    const int8_t* q_in;                     // int8 [M][K]      (contraction-only mode)
    const uint32_t* packed[kGemvMaxProj];   // [N_g][K/16]
    const float* scale[kGemvMaxProj];       // beta_g           (fused mode)
    uint16_t* y[kGemvMaxProj];              // bf16 [M][N_g]    (fused mode)
    int32_t* acc;                           // int32 [M][N]     (contraction-only mode, one projection)
    int row_start[kGemvMaxProj + 1];        // prefix sums of N_g
    float eps;
    int M, K, nproj;
    int rows_per_stage;                     // multiple of kGemvBlockRows
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
    constexpr int B = kGemvBlockRows;
    int rs = B * (kGemvStageTarget / (B * rowbytes));
    if (rs < B) rs = B;
    if (rs > 64) rs = 64;
    int grid = static_cast<int>((R + B - 1) / B);
    if (grid > num_sms) grid = num_sms;
    const int per = static_cast<int>((R + grid - 1) / grid);  // blocks may be partial
    const int want = (per + rs - 1) / rs;  // stages that hold the CTA's whole slab
    // Prefer a ring that holds the whole slab within the two-CTA budget, then
    // fewer stages, then the one-CTA budget, then smaller stages.
    const size_t budgets[2] = {static_cast<size_t>(kGemvSmemTwoCta), static_cast<size_t>(kGemvSmemBudget)};
    for (size_t budget : budgets) {
        for (int r = rs; r >= B; r -= B) {
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

// Fixed-shape pairwise combine of n (a power of two) per-warp partials: the
// same tree every run, so the fp64 sum is deterministic.
template <int n, typename T>
__device__ __forceinline__ T tree_sum(const T* v) {
    if constexpr (n == 1) return v[0];
    else return tree_sum<n / 2>(v) + tree_sum<n / 2>(v + n / 2);
}

template <int n>
__device__ __forceinline__ float tree_max(const float* v) {
    if constexpr (n == 1) return v[0];
    else return fmaxf(tree_max<n / 2>(v), tree_max<n / 2>(v + n / 2));
}

template <int NW>
__device__ __forceinline__ void gemv_compute_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory");
}

// projection of a global row (row_start is short and sorted)
__device__ __forceinline__ int gemv_proj_of(const GemvParams& p, int r) {
    int g = 0;
#pragma unroll
    for (int i = 1; i < kGemvMaxProj; ++i)
        if (i < p.nproj && r >= p.row_start[i]) g = i;
    return g;
}

template <int MT, bool FUSED, bool GLU = false>
__global__ void __launch_bounds__(gemv_threads(MT), gemv_ctas_per_sm(MT)) gemv_kernel(const __grid_constant__ GemvParams p) {
    constexpr int NW = gemv_compute_warps(MT);
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t full_bar[kGemvMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kGemvMaxStages];
    __shared__ __align__(8) uint64_t act_bar;
    __shared__ float deq_s[MT];
    __shared__ float beta_s[kGemvMaxProj];
    __shared__ double red_d[NW];
    __shared__ float red_f[NW];
    __shared__ int red_i[NW];
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

    // shared memory: [ring: S stages][gamma fp32 K][x bf16 M*K][q int8 M*K].
    // q is stored t-major: the 16 codes k = 64c + 16t .. +15 sit at 16*(t*C + c)
    // (C = K/64), so the 8 lanes of a row read 128 contiguous bytes at each t.
    uint8_t* ring = smem;
    float* gamma_s = reinterpret_cast<float*>(smem + static_cast<size_t>(S) * p.stage_bytes);
    uint16_t* x_s = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(gamma_s) + 4 * static_cast<size_t>(K));
    int8_t* q_s = reinterpret_cast<int8_t*>(reinterpret_cast<uint8_t*>(x_s) + 2 * static_cast<size_t>(p.M) * K);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], NW);
        }
        mbar_init(&act_bar, 1);
        abort_flag = 0;
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == NW) {
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
            // gamma and the weights are parameters: fetched before the dependency
            // wait (gamma first, the normalisation needs it before any weight)
            const uint32_t x_bytes = static_cast<uint32_t>((FUSED ? 2 : 1) * static_cast<size_t>(p.M) * K);
            const uint32_t g_bytes = FUSED ? 4u * static_cast<uint32_t>(K) : 0u;
            mbar_arrive_expect_tx(&act_bar, x_bytes + g_bytes);
            if constexpr (FUSED) bulk_g2s(gamma_s, p.gamma, g_bytes, &act_bar);
            const int first = min(nst, S);
            for (int s = 0; s < first; ++s) issue_stage(s);
            // Activations may come from the previous kernel on the stream, so
            // they are read only after it has finished; their lines are brought
            // into L2 now (a prefetch reads nothing into this CTA, and L2 stays
            // coherent with whatever that kernel still writes).
            {
                const uint8_t* xb = FUSED ? reinterpret_cast<const uint8_t*>(p.x) : reinterpret_cast<const uint8_t*>(p.q_in);
                for (uint32_t off = 0; off < x_bytes; off += 65536u)
                    bulk_prefetch_l2(xb + off, x_bytes - off < 65536u ? x_bytes - off : 65536u);
                if constexpr (GLU) {
                    const uint8_t* ub = reinterpret_cast<const uint8_t*>(p.u);
                    for (uint32_t off = 0; off < x_bytes; off += 65536u)
                        bulk_prefetch_l2(ub + off, x_bytes - off < 65536u ? x_bytes - off : 65536u);
                }
            }
            pdl_wait();
            bulk_g2s(x_s, FUSED ? static_cast<const void*>(p.x) : static_cast<const void*>(p.q_in), x_bytes, &act_bar);
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
    // Token m is shared by WPT = NW / MP warps (MP = M rounded up to a power of
    // two); every reduction is per-thread sequential, a warp xor-tree, then the
    // group's warps in index order, so the result does not vary run to run.
    constexpr int MP = MT <= 1 ? 1 : (MT <= 2 ? 2 : (MT <= 4 ? 4 : 8));
    constexpr int WPT = NW / MP;
    const int m = warp / WPT;
    const bool active = m < p.M;
    const int tg = (warp % WPT) * 32 + lane;
    const int w0 = m * WPT;
    if (FUSED && threadIdx.x < p.nproj) beta_s[threadIdx.x] = __ldg(p.scale[threadIdx.x]);  // read after a compute sync
    const bool act_ok = mbar_wait(&act_bar, 0, &abort_flag);
    if constexpr (FUSED) {
        const int C8 = K >> 3;
        uint4* xr = reinterpret_cast<uint4*>(x_s + static_cast<size_t>(m) * K);
        const float4* g4 = reinterpret_cast<const float4*>(gamma_s);
        double s2 = 0.0;
        if (active && act_ok) {
            for (int c = tg; c < C8; c += 32 * WPT) {
                uint4 v = xr[c];
                if constexpr (GLU) {
                    // the GLU gated product replaces x (this thread alone reads chunk c later)
                    v = glu_gate8(v, __ldg(reinterpret_cast<const uint4*>(p.u + static_cast<size_t>(m) * K) + c));
                    xr[c] = v;
                }
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                double sq[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const double lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
                    sq[i] = lo * lo + hi * hi;
                }
                s2 += (sq[0] + sq[1]) + (sq[2] + sq[3]);  // exact sums: the order does not matter
            }
        }
        s2 = warp_sum_f64(s2);
        if (lane == 0) red_d[warp] = s2;
        gemv_compute_sync<NW>();
        s2 = tree_sum<WPT>(red_d + w0);
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
        amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));  // amax >= 0
        if (lane == 0) red_f[warp] = amax;
        gemv_compute_sync<NW>();
        amax = tree_max<WPT>(red_f + w0);
        const float a = fmaxf(amax, 1e-5f);
        const float s = __fdiv_rn(127.0f, a);
        if (active && tg == 0) deq_s[m] = __fdiv_rn(a, 127.0f);  // published by the barrier below

        // codes: v = r * s (|v| <= 127 up to an ulp, as a >= |r|) is rounded to
        // the nearest integer, ties to even, by adding 1.5 * 2^23, which leaves
        // the code in the low byte; the clamp of the definition never acts
        int qs = 0;
        if (active && act_ok) {
            int8_t* qrow = q_s + static_cast<size_t>(m) * K;
            const int C64 = K >> 6;
            for (int c = tg; c < C8; c += 32 * WPT) {
                const uint4 v = xr[c];
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                const float4 ga = g4[2 * c], gb = g4[2 * c + 1];
                const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                uint32_t cb[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float xv =
                        (i & 1) ? __uint_as_float(w[i >> 1] & 0xFFFF0000u) : __uint_as_float(w[i >> 1] << 16);
                    cb[i] = __float_as_uint(__fadd_rn(__fmul_rn(__fmul_rn(__fmul_rn(xv, inv), g[i]), s), 12582912.0f));
                }
                const uint32_t o0 = __byte_perm(__byte_perm(cb[0], cb[1], 0x0040), __byte_perm(cb[2], cb[3], 0x0040), 0x5410);
                const uint32_t o1 = __byte_perm(__byte_perm(cb[4], cb[5], 0x0040), __byte_perm(cb[6], cb[7], 0x0040), 0x5410);
                qs = __dp4a(static_cast<int>(o0), 0x01010101, qs);
                qs = __dp4a(static_cast<int>(o1), 0x01010101, qs);
                // codes k = 8c .. 8c+7 -> unit (c/8, (c%8)/2), half c%2 of the t-major layout
                *reinterpret_cast<uint2*>(qrow + 16 * (((c & 7) >> 1) * C64 + (c >> 3)) + 8 * (c & 1)) =
                    make_uint2(o0, o1);
            }
        }
        qs = __reduce_add_sync(0xffffffffu, qs);
        if (lane == 0) red_i[warp] = qs;
    } else {
        int qs = 0;
        if (active && act_ok) {
            // codes arrive in natural order in the x area; 16-byte unit u = 4c + t
            // moves to position t*C + c of the t-major layout
            const uint4* qr = reinterpret_cast<const uint4*>(reinterpret_cast<const int8_t*>(x_s) +
                                                             static_cast<size_t>(m) * K);
            uint4* qrow = reinterpret_cast<uint4*>(q_s + static_cast<size_t>(m) * K);
            const int C64 = K >> 6;
            for (int c = tg; c < (K >> 4); c += 32 * WPT) {
                const uint4 v = qr[c];
                qrow[(c & 3) * C64 + (c >> 2)] = v;
                qs = __dp4a(static_cast<int>(v.x), 0x01010101, qs);
                qs = __dp4a(static_cast<int>(v.y), 0x01010101, qs);
                qs = __dp4a(static_cast<int>(v.z), 0x01010101, qs);
                qs = __dp4a(static_cast<int>(v.w), 0x01010101, qs);
            }
        }
        qs = __reduce_add_sync(0xffffffffu, qs);
        if (lane == 0) red_i[warp] = qs;
    }
    // codes, per-warp code sums and dequantisation factors visible; the warps
    // agree on whether gamma arrived
    if (!named_barrier_and<1, NW * 32>(act_ok)) return;
    // the sum of the codes of each token, from its warps' partial sums in index order
    int qsum_r[MT];
#pragma unroll
    for (int mm = 0; mm < MT; ++mm) qsum_r[mm] = tree_sum<WPT>(red_i + mm * WPT);

    // ---------------- contraction over the staged rows
    // Blocks of 8 rows go round-robin to the compute warps over the whole slab
    // (for one token and a resident slab, possibly items of 4 rows instead).
    const int rsub = lane >> 3;    // lane handles rows rsub and rsub + 4 of a block
    const int l8 = lane & 7;       // lane within the row
    const int C = K >> 6;          // 16-byte chunks (64 weights) per row
    const int bps = p.rows_per_stage / kGemvBlockRows;
    const int nblocks = (nrows + kGemvBlockRows - 1) / kGemvBlockRows;

    auto finish_row = [&](const int (&ac)[MT][4], int s, int rl, bool valid) {
        const int r = row0 + s * p.rows_per_stage + rl;
        const int g = gemv_proj_of(p, valid ? r : row0);
        const int n = r - p.row_start[g];
        const int Ng = p.row_start[g + 1] - p.row_start[g];
#pragma unroll
        for (int mm = 0; mm < MT; ++mm) {
            int t = ac[mm][0] + (ac[mm][1] >> 2) + (ac[mm][2] >> 4) + (ac[mm][3] >> 6);
            t += __shfl_xor_sync(0xffffffffu, t, 1);
            t += __shfl_xor_sync(0xffffffffu, t, 2);
            t += __shfl_xor_sync(0xffffffffu, t, 4);
            if (valid && l8 == 0 && mm < p.M) {
                const int v = t - qsum_r[mm];
                if constexpr (FUSED) {
                    const float cm = __fmul_rn(deq_s[mm], beta_s[g]);
                    const __nv_bfloat16 yb = __float2bfloat16_rn(__fmul_rn(static_cast<float>(v), cm));
                    p.y[g][static_cast<size_t>(mm) * Ng + n] = __bfloat16_as_ushort(yb);
                } else {
                    p.acc[static_cast<size_t>(mm) * Ng + n] = v;
                }
            }
        }
    };
    auto do_block = [&](int gb, int s, int slot) {
        const int rs = min(p.rows_per_stage, nrows - s * p.rows_per_stage);
        const int b = gb - s * bps;
        const uint8_t* stage = ring + static_cast<size_t>(slot) * p.stage_bytes;
        const int rl0 = kGemvBlockRows * b + rsub, rl1 = rl0 + 4;
        const bool v0 = rl0 < rs, v1 = rl1 < rs;
        int acc0[MT][4], acc1[MT][4];
        const uint4* w0p = reinterpret_cast<const uint4*>(stage + static_cast<size_t>(v0 ? rl0 : 0) * rowbytes);
        const uint4* w1p = reinterpret_cast<const uint4*>(stage + static_cast<size_t>(v1 ? rl1 : 0) * rowbytes);
        if constexpr (MT == 1) {
            // one token: separate accumulators per (row, t, j), 32 independent
            // DP4A chains per lane, summed once after the loop
            int a[2][4][4];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int j = 0; j < 4; ++j) a[h][t][j] = 0;
#pragma unroll 2
            for (int c = l8; c < C; c += 8) {
                const uint4 wa = w0p[c], wb = w1p[c];
                const uint32_t da[4] = {wa.x, wa.y, wa.z, wa.w};
                const uint32_t db[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const uint4 qv = *reinterpret_cast<const uint4*>(q_s + 16 * (t * C + c));
                    a[0][t][0] = dp4a_us(da[t] & 0x03030303u, qv.x, a[0][t][0]);
                    a[0][t][1] = dp4a_us(da[t] & 0x0C0C0C0Cu, qv.y, a[0][t][1]);
                    a[0][t][2] = dp4a_us(da[t] & 0x30303030u, qv.z, a[0][t][2]);
                    a[0][t][3] = dp4a_us(da[t] & 0xC0C0C0C0u, qv.w, a[0][t][3]);
                    a[1][t][0] = dp4a_us(db[t] & 0x03030303u, qv.x, a[1][t][0]);
                    a[1][t][1] = dp4a_us(db[t] & 0x0C0C0C0Cu, qv.y, a[1][t][1]);
                    a[1][t][2] = dp4a_us(db[t] & 0x30303030u, qv.z, a[1][t][2]);
                    a[1][t][3] = dp4a_us(db[t] & 0xC0C0C0C0u, qv.w, a[1][t][3]);
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc0[0][j] = (a[0][0][j] + a[0][1][j]) + (a[0][2][j] + a[0][3][j]);
                acc1[0][j] = (a[1][0][j] + a[1][1][j]) + (a[1][2][j] + a[1][3][j]);
            }
        } else {
#pragma unroll
        for (int mm = 0; mm < MT; ++mm)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc0[mm][j] = acc1[mm][j] = 0;
#pragma unroll 2
        for (int c = l8; c < C; c += 8) {
            const uint4 wa = w0p[c], wb = w1p[c];
            const uint32_t da[4] = {wa.x, wa.y, wa.z, wa.w};
            const uint32_t db[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const uint32_t a0 = da[t] & 0x03030303u, a1 = da[t] & 0x0C0C0C0Cu;
                const uint32_t a2 = da[t] & 0x30303030u, a3 = da[t] & 0xC0C0C0C0u;
                const uint32_t c0 = db[t] & 0x03030303u, c1 = db[t] & 0x0C0C0C0Cu;
                const uint32_t c2 = db[t] & 0x30303030u, c3 = db[t] & 0xC0C0C0C0u;
#pragma unroll
                for (int mm = 0; mm < MT; ++mm) {
                    const uint4 qv =
                        *reinterpret_cast<const uint4*>(q_s + static_cast<size_t>(mm) * K + 16 * (t * C + c));
                    acc0[mm][0] = dp4a_us(a0, qv.x, acc0[mm][0]);
                    acc0[mm][1] = dp4a_us(a1, qv.y, acc0[mm][1]);
                    acc0[mm][2] = dp4a_us(a2, qv.z, acc0[mm][2]);
                    acc0[mm][3] = dp4a_us(a3, qv.w, acc0[mm][3]);
                    acc1[mm][0] = dp4a_us(c0, qv.x, acc1[mm][0]);
                    acc1[mm][1] = dp4a_us(c1, qv.y, acc1[mm][1]);
                    acc1[mm][2] = dp4a_us(c2, qv.z, acc1[mm][2]);
                    acc1[mm][3] = dp4a_us(c3, qv.w, acc1[mm][3]);
                }
            }
        }
        }
        finish_row(acc0, s, rl0, v0);
        finish_row(acc1, s, rl1, v1);
    };

    // One token, whole slab resident: items of 4 rows (lane group rsub takes
    // row rsub), so a slab of few rows spreads over more warps.
    auto do_rows4 = [&](int it) {
        const int s = (4 * it) / p.rows_per_stage;
        const int rs = min(p.rows_per_stage, nrows - s * p.rows_per_stage);
        const int rl = 4 * it - s * p.rows_per_stage + rsub;
        const bool v = rl < rs;
        const uint4* wp = reinterpret_cast<const uint4*>(ring + static_cast<size_t>(s) * p.stage_bytes +
                                                         static_cast<size_t>(v ? rl : 0) * rowbytes);
        int a[4][4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int j = 0; j < 4; ++j) a[t][j] = 0;
#pragma unroll 2
        for (int c = l8; c < C; c += 8) {
            const uint4 wa = wp[c];
            const uint32_t da[4] = {wa.x, wa.y, wa.z, wa.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const uint4 qv = *reinterpret_cast<const uint4*>(q_s + 16 * (t * C + c));
                a[t][0] = dp4a_us(da[t] & 0x03030303u, qv.x, a[t][0]);
                a[t][1] = dp4a_us(da[t] & 0x0C0C0C0Cu, qv.y, a[t][1]);
                a[t][2] = dp4a_us(da[t] & 0x30303030u, qv.z, a[t][2]);
                a[t][3] = dp4a_us(da[t] & 0xC0C0C0C0u, qv.w, a[t][3]);
            }
        }
        int acc[MT][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[0][j] = (a[0][j] + a[1][j]) + (a[2][j] + a[3][j]);
        finish_row(acc, s, rl, v);
    };

    if (nst <= S) {
        // The ring holds the whole slab: every slot is filled once (phase 0),
        // so a warp waits only for the stage of each of its blocks.
        // one token: 4-row items when 8-row blocks would leave warps idle and the
        // busiest warp gets fewer rows
        const int n4 = (nrows + 3) / 4;
        bool rows4 = false;
        if constexpr (MT == 1) rows4 = nblocks < NW && (n4 + NW - 1) / NW * 4 < kGemvBlockRows;
        if (rows4) {
            if constexpr (MT == 1) {
                for (int it = warp; it < n4; it += NW) {
                    if (!mbar_wait(&full_bar[(4 * it) / p.rows_per_stage], 0, &abort_flag)) break;
                    do_rows4(it);
                }
            }
        } else {
            for (int gb = warp; gb < nblocks; gb += NW) {
                const int s = gb / bps;
                if (!mbar_wait(&full_bar[s], 0, &abort_flag)) break;
                do_block(gb, s, s);
            }
        }
    } else {
        // Slots are refilled: every warp walks the stages in order and releases
        // each one (a parity wait only tells adjacent phases apart, so no warp
        // may look at a slot more than one phase ahead of its last release).
        for (int s = 0; s < nst; ++s) {
            const int slot = s % S;
            if (!mbar_wait(&full_bar[slot], (s / S) & 1, &abort_flag)) break;
            const int nb = (min(p.rows_per_stage, nrows - s * p.rows_per_stage) + kGemvBlockRows - 1) / kGemvBlockRows;
            int first = warp - (s * bps) % NW;  // first block of this stage owned by this warp
            if (first < 0) first += NW;
            for (int b = first; b < nb; b += NW) do_block(s * bps + b, s, slot);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[slot]);
        }
    }
}

}  // namespace mmf
