// gemv_tc.cuh -- decode-regime contraction for a few tokens (9 <= M <= 32) on
// the 5th-generation tensor cores.
//
// With M tokens the add/sub contraction on CUDA cores costs about M/4 integer
// instructions per weight (one DP4A per four weights per token), so beyond a
// token or two it, not HBM, sets the time.  Here the weights are unpacked once
// per K chunk into an int8 tile and the tokens' codes ride along as the MMA's
// B operand, so a weight costs the same however many tokens there are.  The
// ternary rule (ld246.com, section "三值权重的应用") is kept as in the other
// kernels: the codes c = w~ + 1 multiply q, and the epilogue subtracts the
// token's sum of q.
//
// Work split as in the CUDA-core decode kernel: the projections of a group
// (sharing x) form one row space, and each CTA owns a slab of at most 128
// consecutive rows (the MMA's M = 128 side; rows past the slab are zero).
// The slab's packed weights are copied into shared memory whole, before the
// dependency wait (programmatic dependent launch), so they stream in while the
// previous kernel runs.  The codes come from the quantiser launched just
// before, written in the MMA's B layout (see the quantiser's blayout mode):
// per 128-wide K chunk, NT token rows of 128 bytes in 8-row 1024-byte
// 128-byte-swizzled atoms; they are copied chunk by chunk into a ring.
// Warp roles (14 warps):
//   warp 0      producer: bulk copies of the weight slab, then (after the
//               dependency wait) of the code chunks
//   warp 1      TMEM allocation (32 columns); lane 0 issues tcgen05.mma
//               (4 x K = 32 per chunk) and the commits
//   warps 4-7   epilogue: tcgen05.ld of the 128 x NT accumulator, subtract
//               sum q, rescale, bf16 y (a warp's 32 lanes = 32 rows)
//   warps 8-15  unpack: 2-bit codes of the slab -> int8 A tiles
// The unpack warps and the MMA thread hand over units of two chunks (a
// barrier wait costs about as much as issuing four small MMAs): per unit the
// unpack warps write two A tiles, make sure the unit's code chunks have
// landed, and signal the unit full once; the MMA thread waits once, issues 8
// MMAs and commits the unit's A slot and its two code slots.
// Every wait is bounded; on timeout the CTA records the error, drains its
// copies and MMAs, frees TMEM and exits.
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kGtRows = 128;                 // A rows per CTA (MMA M)
constexpr int kGtThreads = 16 * 32;
constexpr int kGtUnpackThreads = 256;        // warps 8-15
constexpr int kGtASlots = 4;                 // unpacked weight chunks in flight
constexpr int kGtUnit = 2;                   // chunks per unpack/MMA hand-over
constexpr int kGtUnits = kGtASlots / kGtUnit;
constexpr int kGtMaxBSlots = 32;
constexpr int kGtMaxProj = 8;
constexpr int kGtSmemBudget = 220 * 1024;

struct GemvTcParams {
    const int8_t* codes;                      // B layout: [K/128][NT/8][8][128 B], swizzled
    const float* absmax;                      // [M]  (fused mode)
    const int* qsum;                          // [M]
    const uint32_t* packed[kGtMaxProj];       // [N_g][K/16]
    const float* scale[kGtMaxProj];           // beta_g      (fused mode)
    uint16_t* y[kGtMaxProj];                  // bf16 [M][N_g] (fused mode)
    int32_t* acc;                             // int32 [M][N] (contraction-only mode, one projection)
    int row_start[kGtMaxProj + 1];
    int nproj;
    int M, K;
    int rows_per_cta;                         // <= 128
    int b_slots;                              // code chunks in flight (<= kGtMaxBSlots)
};

struct GemvTcPlan {
    int rows_per_cta, grid, b_slots;
    size_t smem_bytes;
};

// Shared memory: [A slots: 4 x 16 KB][B slots: b_slots x NT*128][weight slab: rows x K/4]
inline size_t gemv_tc_smem(int NT, int rows, int K, int b_slots) {
    return static_cast<size_t>(kGtASlots) * kGtRows * 128 + static_cast<size_t>(b_slots) * NT * 128 +
           static_cast<size_t>(rows) * (K / 4) + 1024;
}

// Host-side launch shape; false if a slab of even 8 rows does not fit.  The
// slab spreads the rows over the SMs (at most 128 a CTA); the ring holds as
// many code chunks as fit (all of them if possible: they come from L2, and
// each copy's latency is paid once per ring turn).  One CTA per SM: under
// programmatic launch the CTAs sit beside the quantiser's, not beside the
// previous contraction's.
inline bool gemv_tc_plan(int NT, int K, int64_t R, int num_sms, GemvTcPlan* plan) {
    const int nchunks = K / 128;
    int rows = static_cast<int>((R + num_sms - 1) / num_sms);
    rows = (rows + 7) & ~7;
    if (rows > kGtRows) rows = kGtRows;
    const int want = nchunks < kGtMaxBSlots ? nchunks : kGtMaxBSlots;
    for (int r = rows; r >= 8; r -= 8) {
        for (int slots = want; slots >= 1; --slots) {
            if (slots < 4 && slots < want) break;
            if (gemv_tc_smem(NT, r, K, slots) <= static_cast<size_t>(kGtSmemBudget)) {
                plan->rows_per_cta = r;
                plan->b_slots = slots;
                plan->grid = static_cast<int>((R + r - 1) / r);
                plan->smem_bytes = gemv_tc_smem(NT, r, K, slots);
                return true;
            }
        }
    }
    return false;
}

__device__ __forceinline__ int gemv_tc_proj_of(const GemvTcParams& p, int r) {
    int g = 0;
#pragma unroll
    for (int i = 1; i < kGtMaxProj; ++i)
        if (i < p.nproj && r >= p.row_start[i]) g = i;
    return g;
}

template <int NT, bool FUSED>
__global__ void __launch_bounds__(kGtThreads, 1) gemv_tc_kernel(const __grid_constant__ GemvTcParams p) {
    static_assert(NT == 16 || NT == 32, "MMA N is 16 or 32 tokens");
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t w_bar;
    __shared__ __align__(8) uint64_t a_full[kGtUnits];
    __shared__ __align__(8) uint64_t a_empty[kGtUnits];
    __shared__ __align__(8) uint64_t b_full[kGtMaxBSlots];
    __shared__ __align__(8) uint64_t b_empty[kGtMaxBSlots];
    __shared__ __align__(8) uint64_t d_full;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_flag;
    __shared__ float deq_s[32];
    __shared__ int qsum_s[32];
    __shared__ float beta_s[kGtMaxProj];

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int kABytes = kGtRows * 128;
    constexpr int kBBytes = NT * 128;
    const int S = p.b_slots;
    uint8_t* a_base = smem;
    uint8_t* b_base = smem + kGtASlots * kABytes;
    uint8_t* w_s = b_base + static_cast<size_t>(S) * kBBytes;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int K = p.K;
    const int rowbytes = K >> 2;
    const int nchunks = K >> 7;
    const int R = p.row_start[p.nproj];
    const int row0 = blockIdx.x * p.rows_per_cta;
    const int nrows = min(R - row0, p.rows_per_cta);
    if (nrows <= 0) return;  // uniform for the CTA, before any barrier

    if (threadIdx.x == 0) {
        mbar_init(&w_bar, 1);
        for (int s = 0; s < kGtUnits; ++s) {
            mbar_init(&a_full[s], kGtUnpackThreads);
            mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < S; ++s) {
            mbar_init(&b_full[s], 1);
            mbar_init(&b_empty[s], 1);
        }
        mbar_init(&d_full, 1);
        abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_s, 32);
        tmem_relinquish();
    }
    if (FUSED && threadIdx.x < p.nproj) beta_s[threadIdx.x] = __ldg(p.scale[threadIdx.x]);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            // the weight slab: parameters, fetched before the dependency wait
            mbar_arrive_expect_tx(&w_bar, static_cast<uint32_t>(nrows) * rowbytes);
            for (int r = row0; r < row0 + nrows;) {  // split at projection boundaries
                const int g = gemv_tc_proj_of(p, r);
                const int e = min(row0 + nrows, p.row_start[g + 1]);
                const uint8_t* src =
                    reinterpret_cast<const uint8_t*>(p.packed[g]) + static_cast<size_t>(r - p.row_start[g]) * rowbytes;
                bulk_g2s(w_s + static_cast<size_t>(r - row0) * rowbytes, src, static_cast<uint32_t>(e - r) * rowbytes,
                         &w_bar);
                r = e;
            }
            // the codes come from the quantiser launched just before
            pdl_wait();
            pdl_launch_dependents();
            int c = 0;
            for (; c < nchunks; ++c) {
                const int s = c % S;
                if (c >= S && !mbar_wait(&b_empty[s], ((c / S) - 1) & 1, &abort_flag)) break;
                mbar_arrive_expect_tx(&b_full[s], kBBytes);
                bulk_g2s(b_base + s * kBBytes, p.codes + static_cast<size_t>(c) * kBBytes, kBBytes, &b_full[s]);
            }
            int zero = 0;
            mbar_wait(&w_bar, 0, &zero);
            for (int u = max(0, c - S); u < c; ++u) mbar_wait(&b_full[u % S], (u / S) & 1, &zero);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kGtRows, NT);
            bool issued = false;
            const int nunits = (nchunks + kGtUnit - 1) / kGtUnit;
            for (int u = 0; u < nunits; ++u) {
                const int su = u % kGtUnits;
                // a full unit also means its code chunks have landed (the unpack warps waited)
                if (!mbar_wait(&a_full[su], (u / kGtUnits) & 1, &abort_flag)) break;
                tc_fence_after();
                const int c0 = kGtUnit * u, c1 = min(c0 + kGtUnit, nchunks);
                for (int c = c0; c < c1; ++c) {
                    const uint32_t a0 = smem_u32(a_base + (kGtUnit * su + c - c0) * kABytes);
                    const uint32_t b0 = smem_u32(b_base + (c % S) * kBBytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_i8(tmem_base, sw128_kmajor_desc(a0 + 32 * kk), sw128_kmajor_desc(b0 + 32 * kk), idesc,
                               (c | kk) != 0 ? 1u : 0u);
                }
                issued = true;
                mma_commit(&a_empty[su]);
                for (int c = c0; c < c1; ++c) mma_commit(&b_empty[c % S]);
            }
            if (issued) mma_commit(&d_full);
            if (issued && abort_flag) {  // d_full may never be waited on: let the MMAs drain here
                int zero = 0;
                mbar_wait(&d_full, 0, &zero);
            }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ unpack
        const int t = threadIdx.x - 8 * 32;  // 0 .. 255
        const int row = t & 127, half = t >> 7;
        // rows past the slab stay zero in every A slot
        if (row >= nrows) {
#pragma unroll
            for (int s = 0; s < kGtASlots; ++s) {
                uint8_t* arow = a_base + s * kABytes + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    *reinterpret_cast<uint4*>(arow + ((4 * half + u) << 4)) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        const bool got_w = mbar_wait(&w_bar, 0, &abort_flag);
        const int nunits = (nchunks + kGtUnit - 1) / kGtUnit;
        for (int u = 0; u < nunits && got_w; ++u) {
            const int su = u % kGtUnits;
            if (u >= kGtUnits && !mbar_wait(&a_empty[su], ((u / kGtUnits) - 1) & 1, &abort_flag)) break;
            const int c0 = kGtUnit * u, c1 = min(c0 + kGtUnit, nchunks);
            for (int c = c0; c < c1 && row < nrows; ++c) {
                const int sa = kGtUnit * su + c - c0;
                // words 4 half .. 4 half + 3 of the chunk: K bytes 16 (4 half + i) .. + 15
                const uint4 wv = *reinterpret_cast<const uint4*>(w_s + static_cast<size_t>(row) * rowbytes + 32 * c +
                                                                 16 * half);
                const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
                uint8_t* arow = a_base + sa * kABytes + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t w = words[i];
                    const uint4 o = make_uint4(w & 0x03030303u, (w >> 2) & 0x03030303u, (w >> 4) & 0x03030303u,
                                               (w >> 6) & 0x03030303u);
                    *reinterpret_cast<uint4*>(arow + (((4 * half + i) ^ (row & 7)) << 4)) = o;
                }
            }
            fence_proxy_async_smem();
            // the unit's code chunks: landed before the unit is signalled full
            bool bok = true;
            if (lane < c1 - c0) bok = mbar_wait(&b_full[(c0 + lane) % S], ((c0 + lane) / S) & 1, &abort_flag);
            if (!__all_sync(0xffffffffu, bok)) break;
            mbar_arrive(&a_full[su]);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        const int wq = warp & 3;
        pdl_wait();  // sums and scales of the codes (also ordered by the MMA barriers)
        if (threadIdx.x - 128 < p.M) {
            const int tt = threadIdx.x - 128;
            qsum_s[tt] = p.qsum[tt];
            if constexpr (FUSED) deq_s[tt] = __fdiv_rn(p.absmax[tt], 127.0f);
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const bool got = mbar_wait(&d_full, 0, &abort_flag);
        if (__all_sync(0xffffffffu, got)) {
            tc_fence_after();
            uint32_t r[32];
            tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * wq) << 16), r);
            tmem_ld_wait();
            const int rl = 32 * wq + lane;
            if (rl < nrows) {
                const int rg = row0 + rl;
                const int g = gemv_tc_proj_of(p, rg);
                const int n = rg - p.row_start[g];
                const int Ng = p.row_start[g + 1] - p.row_start[g];
#pragma unroll
                for (int tt = 0; tt < NT; ++tt) {
                    if (tt < p.M) {
                        const int v = static_cast<int>(r[tt]) - qsum_s[tt];
                        if constexpr (FUSED) {
                            const float cm = __fmul_rn(deq_s[tt], beta_s[g]);
                            const __nv_bfloat16 yb = __float2bfloat16_rn(__fmul_rn(static_cast<float>(v), cm));
                            p.y[g][static_cast<size_t>(tt) * Ng + n] = __bfloat16_as_ushort(yb);
                        } else {
                            p.acc[static_cast<size_t>(tt) * Ng + n] = v;
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 32);
    }
}

}  // namespace mmf
