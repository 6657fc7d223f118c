// gemm_tc.cuh -- large-M ternary contraction on the 5th-generation tensor
// cores (tcgen05, kind::i8, int32 accumulators in TMEM).
//
// The product with ternary weights is a dense contraction at large M, so it
// runs as one: the 2-bit weight codes c = w~ + 1 are unpacked to int8 in
// shared memory and multiplied with the int8 activation codes; the epilogue
// subtracts the per-token sum of q, which turns sum_k c q into
// sum_k w~ q = (sum over w~=+1 of q) - (sum over w~=-1 of q)
// (the ternary accumulation of ld246.com, section "三值权重的应用").
//
// Tile: 128 weight rows (MMA M) x BT tokens (MMA N), K in stages of 128; the
// weights are the A operand, so one unpacked weight tile feeds BT tokens.
// Persistent: one CTA per SM walks the tiles (token tile major, weight tile
// minor, so CTAs working at the same time share activation tiles in L2), with
// two TMEM accumulators so a tile's epilogue overlaps the next tile's MMAs.
// When the tiles end in a partial wave of R tiles with 2R <= the grid, those
// tiles become 2R items of BT / 2 tokens each (an N = BT / 2 MMA on the first
// half of the loaded token tile), so the last wave takes half a tile's time.
// Warp roles (640 threads):
//   warp 0      TMA producer: q tile (BT x 128 B, 128-byte swizzle) and the
//               packed weight tile (128 x 32 B) per stage
//   warp 1      TMEM allocation; lane 0 issues tcgen05.mma (4 x K=32 per
//               stage) and the tcgen05.commits
//   warps 4-15  epilogue, three warps per TMEM sub-partition (a warp reaches
//               the 32 TMEM lanes of sub-partition warp % 4) taking every
//               third 32-token chunk: tcgen05.ld, subtract sum q, rescale,
//               transpose through shared memory, 16-byte stores of y
//   warps 16-19 unpack: thread u expands row u's 128 codes to int8 in the
//               128-byte-swizzled K-major layout the MMA reads
// Every wait is bounded; on timeout the CTA records the error, drains its
// copies and MMAs, frees TMEM and exits.
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kTcRows = 128;      // weight rows per tile (MMA M)
constexpr int kTcK = 128;         // K (bytes of int8) per stage
constexpr int kTcStages = 4;
constexpr int kTcEpiWarps = 12;                        // three per TMEM sub-partition
constexpr int kTcThreads = (8 + kTcEpiWarps) * 32;     // warps 0-3 TMA/MMA/idle, epilogue, 4 unpack
constexpr int kTcPackedBytes = kTcRows * (kTcK / 4);  // 4 KB of 2-bit codes per stage
constexpr int kTcEpiBarrier = 2;                       // named barrier of the epilogue warps

template <int BT>
struct TcLayout {
    static constexpr int a_bytes = kTcRows * kTcK;  // 16 KB
    static constexpr int b_bytes = BT * kTcK;
    static constexpr int stage_bytes = a_bytes + b_bytes + kTcPackedBytes;
    static constexpr int epi_bytes = kTcEpiWarps * 16 * 32 * 2;  // per-warp 16 x 32 bf16 transpose tiles
    static constexpr int smem_bytes = kTcStages * stage_bytes + epi_bytes + 1024;  // + alignment slack
    static constexpr int acc_cols = BT < 32 ? 32 : BT;
    static constexpr int tmem_cols = 2 * acc_cols;  // double-buffered accumulator
};

struct TcParams {
    const int* qsum;        // [M]
    const float* absmax;    // [M]      (fused mode)
    const float* scale;     // beta     (fused mode)
    uint16_t* y;            // bf16 [M][N]
    int32_t* acc;           // int32 [M][N]
    int M, K, N;
    int n_tiles;            // ceil(N / 128)
    int num_tiles;          // n_tiles * ceil(M / BT)
    // work items: the first full_items are whole tiles; each tile after them
    // (the last, partial wave) is two items of BT / 2 tokens (BT = 256 only)
    int full_items;
    int num_items;
};

template <int BT, bool FUSED>
__global__ void __launch_bounds__(kTcThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_w,
                   const TcParams p) {
    using L = TcLayout<BT>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kTcStages];
    __shared__ __align__(8) uint64_t unpacked_bar[kTcStages];
    __shared__ __align__(8) uint64_t empty_bar[kTcStages];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_flag;
    __shared__ __align__(16) int qsum_s[BT < 16 ? 16 : BT];
    __shared__ __align__(16) float cm_s[BT < 16 ? 16 : BT];

    // 1024-byte aligned base (128-byte swizzle atoms are 8 rows x 128 B)
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    auto a_tile = [&](int s) { return smem + s * L::stage_bytes; };
    auto b_tile = [&](int s) { return smem + s * L::stage_bytes + L::a_bytes; };
    auto p_tile = [&](int s) { return smem + s * L::stage_bytes + L::a_bytes + L::b_bytes; };
    uint16_t* epi_tile = reinterpret_cast<uint16_t*>(smem + kTcStages * L::stage_bytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = p.K / kTcK;
    const int G = gridDim.x;
    // work item -> weight rows n0.., tokens t0 .. t0 + ntok - 1
    auto item_at = [&](int it, int& n0, int& t0, int& ntok) {
        int tile = it, hv = 0;
        ntok = BT;
        if (it >= p.full_items) {
            tile = p.full_items + ((it - p.full_items) >> 1);
            hv = (it - p.full_items) & 1;
            ntok = BT / 2;
        }
        n0 = (tile % p.n_tiles) * kTcRows;
        t0 = (tile / p.n_tiles) * BT + hv * (BT / 2);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&unpacked_bar[s], 128);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], kTcEpiWarps);
        }
        mbar_init(&drain_bar, 1);
        abort_flag = 0;
        mbar_fence_init();
        prefetch_tensormap(&tmap_q);
        prefetch_tensormap(&tmap_w);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_s, L::tmem_cols);
        tmem_relinquish();
    }
    // the codes, sums and scales come from the kernel before (no-op unless
    // launched as a programmatic dependent)
    pdl_wait();
    pdl_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int g = 0;  // stage uses so far
            bool ok = true;
            for (int it = blockIdx.x; it < p.num_items && ok; it += G) {
                int n0, t0, ntok;
                item_at(it, n0, t0, ntok);  // a half item loads the whole box from t0 (rows past M read zero)
                for (int ks = 0; ks < nk; ++ks, ++g) {
                    const int s = g % kTcStages;
                    if (g >= kTcStages && !mbar_wait(&empty_bar[s], ((g / kTcStages) - 1) & 1, &abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full_bar[s], L::b_bytes + kTcPackedBytes);
                    tma_load_2d(b_tile(s), &tmap_q, ks * kTcK, t0, &full_bar[s]);
                    tma_load_2d(p_tile(s), &tmap_w, ks * (kTcK / 4), n0, &full_bar[s]);
                }
            }
            // Let every copy this CTA started land before the CTA can exit.
            int zero = 0;
            for (int u = max(0, g - kTcStages); u < g; ++u)
                mbar_wait(&full_bar[u % kTcStages], (u / kTcStages) & 1, &zero);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_full = idesc_i8(kTcRows, BT);
            constexpr uint32_t idesc_half = BT == 256 ? idesc_i8(kTcRows, BT / 2) : idesc_full;
            bool issued_any = false, ok = true;
            int g = 0, li = 0;
            for (int it = blockIdx.x; it < p.num_items && ok; it += G, ++li) {
                const uint32_t idesc = it < p.full_items ? idesc_full : idesc_half;  // N = the item's tokens
                const int buf = li & 1;
                if (li >= 2 && !mbar_wait(&tempty_bar[buf], ((li >> 1) - 1) & 1, &abort_flag)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(buf * L::acc_cols);
                for (int ks = 0; ks < nk; ++ks, ++g) {
                    const int s = g % kTcStages;
                    const uint32_t par = (g / kTcStages) & 1;
                    if (!mbar_wait(&full_bar[s], par, &abort_flag) || !mbar_wait(&unpacked_bar[s], par, &abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(a_tile(s)), b0 = smem_u32(b_tile(s));
#pragma unroll
                    for (int kk = 0; kk < kTcK / 32; ++kk)
                        mma_i8(d, sw128_kmajor_desc(a0 + 32 * kk), sw128_kmajor_desc(b0 + 32 * kk), idesc,
                               (ks | kk) != 0 ? 1u : 0u);
                    issued_any = true;
                    mma_commit(&empty_bar[s]);
                }
                if (ok) mma_commit(&tfull_bar[buf]);
            }
            if (issued_any) {
                mma_commit(&drain_bar);
                int zero = 0;
                mbar_wait(&drain_bar, 0, &zero);
            }
        }
    } else if (warp >= 4 + kTcEpiWarps) {
        // ------------------------------------------------------------ unpack
        const int u = threadIdx.x - (4 + kTcEpiWarps) * 32;  // weight row within the tile
        int g = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < p.num_items && ok; it += G) {
            for (int ks = 0; ks < nk; ++ks, ++g) {
                const int s = g % kTcStages;
                if (!mbar_wait(&full_bar[s], (g / kTcStages) & 1, &abort_flag)) {
                    ok = false;
                    break;
                }
                const uint4* prow = reinterpret_cast<const uint4*>(p_tile(s) + u * (kTcK / 4));
                const uint4 pa = prow[0], pb = prow[1];
                const uint32_t words[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
                uint8_t* arow = a_tile(s) + (u >> 3) * 1024 + (u & 7) * 128;
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    // word t holds K bytes 16t .. 16t+15 of this stage; byte-lane j of
                    // the output chunk gets codes 4j .. 4j+3 (bits 2j of each byte)
                    const uint32_t w = words[t];
                    uint4 o;
                    o.x = w & 0x03030303u;
                    o.y = (w >> 2) & 0x03030303u;
                    o.z = (w >> 4) & 0x03030303u;
                    o.w = (w >> 6) & 0x03030303u;
                    *reinterpret_cast<uint4*>(arow + ((t ^ (u & 7)) << 4)) = o;
                }
                fence_proxy_async_smem();
                mbar_arrive(&unpacked_bar[s]);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        const int wq = warp & 3;                    // TMEM lanes 32*wq .. 32*wq+31 (a warp's sub-partition)
        const int half = (warp - 4) >> 2;           // which of the warps of that sub-partition
        const int et = threadIdx.x - 128;           // 0 .. 32*kTcEpiWarps-1
        uint16_t* stg = epi_tile + (warp - 4) * (16 * 32);  // [16 tokens][32 rows] bf16
        const bool vec_ok = FUSED && (p.N % 8) == 0;
        int li = 0;
        for (int it = blockIdx.x; it < p.num_items; it += G, ++li) {
            const int buf = li & 1;
            int n0, t0, ntok;
            item_at(it, n0, t0, ntok);
            // per-token constants of this tile (the previous tile's are no longer read)
            asm volatile("bar.sync %0, %1;" ::"n"(kTcEpiBarrier), "n"(kTcEpiWarps * 32) : "memory");
            for (int i = et; i < ntok; i += kTcEpiWarps * 32) {
                const int t = t0 + i;
                int qs = 0;
                float cm = 0.0f;
                if (t < p.M) {
                    qs = p.qsum[t];
                    if constexpr (FUSED) cm = __fmul_rn(__fdiv_rn(p.absmax[t], 127.0f), __ldg(p.scale));
                }
                qsum_s[i] = qs;
                cm_s[i] = cm;
            }
            // the epilogue warps leave together or not at all (they share a named barrier)
            const bool got = mbar_wait(&tfull_bar[buf], (li >> 1) & 1, &abort_flag);
            if (!named_barrier_and<kTcEpiBarrier, kTcEpiWarps * 32>(got)) break;
            tc_fence_after();
            const int n = n0 + 32 * wq + lane;
            const int chunks = BT < 32 ? 1 : ntok / 32;
            constexpr int kCols = BT < 32 ? BT : 32;
#pragma unroll 1
            for (int cc = half; cc < chunks; cc += kTcEpiWarps / 4) {
                uint32_t r[32];
                const uint32_t taddr = tmem_base + static_cast<uint32_t>(buf * L::acc_cols) +
                                       (static_cast<uint32_t>(32 * wq) << 16) + 32 * cc;
                tmem_ld_32x32b_x32(taddr, r);
                tmem_ld_wait();
                if (vec_ok) {
                    // 16 tokens at a time through the transpose tile, as bf16 pairs:
                    // word (pair i/2, row lane) holds tokens i and i+1 of this lane's row
                    uint32_t* stg32 = reinterpret_cast<uint32_t*>(stg);
#pragma unroll
                    for (int h = 0; h < (kCols + 15) / 16; ++h) {
#pragma unroll
                        for (int i8 = 0; i8 < 16 && 16 * h + i8 < kCols; i8 += 8) {
                            // per-token constants, 8 tokens per pair of broadcast 16-byte loads
                            const int tb = 32 * cc + 16 * h + i8;
                            const int4 qa = *reinterpret_cast<const int4*>(qsum_s + tb);
                            const int4 qb = *reinterpret_cast<const int4*>(qsum_s + tb + 4);
                            const float4 ca = *reinterpret_cast<const float4*>(cm_s + tb);
                            const float4 cb = *reinterpret_cast<const float4*>(cm_s + tb + 4);
                            const int qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
                            const float cv[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
#pragma unroll
                            for (int k = 0; k < 8; k += 2) {
                                const int v0 = static_cast<int>(r[16 * h + i8 + k]) - qv[k];
                                const int v1 = static_cast<int>(r[16 * h + i8 + k + 1]) - qv[k + 1];
                                const __nv_bfloat162 y2 = __floats2bfloat162_rn(__fmul_rn(static_cast<float>(v0), cv[k]),
                                                                                __fmul_rn(static_cast<float>(v1), cv[k + 1]));
                                stg32[((i8 + k) >> 1) * 32 + lane] = *reinterpret_cast<const uint32_t*>(&y2);
                            }
                        }
                        __syncwarp();
                        // lane: token pair lane/4, rows 8*(lane%4) .. +7 -> two 16-byte stores
                        {
                            const int pr = lane >> 2;
                            const int nr = n0 + 32 * wq + 8 * (lane & 3);
                            const uint4 wa = *reinterpret_cast<const uint4*>(stg32 + pr * 32 + 8 * (lane & 3));
                            const uint4 wb = *reinterpret_cast<const uint4*>(stg32 + pr * 32 + 8 * (lane & 3) + 4);
                            const uint4 even = make_uint4(__byte_perm(wa.x, wa.y, 0x5410), __byte_perm(wa.z, wa.w, 0x5410),
                                                          __byte_perm(wb.x, wb.y, 0x5410), __byte_perm(wb.z, wb.w, 0x5410));
                            const uint4 odd = make_uint4(__byte_perm(wa.x, wa.y, 0x7632), __byte_perm(wa.z, wa.w, 0x7632),
                                                         __byte_perm(wb.x, wb.y, 0x7632), __byte_perm(wb.z, wb.w, 0x7632));
                            const int i = 16 * h + 2 * pr;
                            const int t = t0 + 32 * cc + i;
                            if (i < kCols && nr < p.N) {
                                if (t < p.M) *reinterpret_cast<uint4*>(p.y + static_cast<size_t>(t) * p.N + nr) = even;
                                if (t + 1 < p.M) *reinterpret_cast<uint4*>(p.y + static_cast<size_t>(t + 1) * p.N + nr) = odd;
                            }
                        }
                        __syncwarp();
                    }
                } else if (n < p.N) {
#pragma unroll
                    for (int i = 0; i < kCols; ++i) {
                        const int ti = 32 * cc + i;
                        const int t = t0 + ti;
                        if (t < p.M) {
                            const int v = static_cast<int>(r[i]) - qsum_s[ti];
                            if constexpr (FUSED) {
                                const __nv_bfloat16 yb =
                                    __float2bfloat16_rn(__fmul_rn(static_cast<float>(v), cm_s[ti]));
                                p.y[static_cast<size_t>(t) * p.N + n] = __bfloat16_as_ushort(yb);
                            } else {
                                p.acc[static_cast<size_t>(t) * p.N + n] = v;
                            }
                        }
                    }
                }
            }
            // this accumulator may be overwritten by the tile after next
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty_bar[buf]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, L::tmem_cols);
    }
}

}  // namespace mmf
