// gemv_wide.cuh -- decode-regime contraction for a few tokens (4 <= M <= 32)
// on the 5th-generation tensor cores, with the weights as the MMA's wide side.
//
// A tcgen05.mma of kind::i8 takes the tensor pipe a time that follows N x K
// (about 28 ns at N = 16..32, about 66 ns at N = 256, K = 32, for M = 64 and
// 128 alike), and every barrier wait costs its thread about 100 ns.  With the
// tokens as N an MMA covers 128 weight rows x 32 K = 4096 weights; here the
// weights are the N = 256 side and the tokens' codes the first rows of the
// M = 128 side, so an MMA covers 256 x 32 = 8192 weights.
// The ternary rule (ld246.com, section "三值权重的应用") is as in the other
// kernels: codes c = w~ + 1 multiply q, and the epilogue subtracts sum q.
//
// Work split: each projection of a group (sharing x) is cut into slabs of 256
// consecutive rows (the last one partial), and each slab's K range is split
// over the ksplit CTAs of a thread-block cluster so the SMs fill (the slabs
// are few at decode sizes).  Each CTA holds its slab's packed weights for its
// K range (a tensor copy of 256 rows per 128-wide K chunk, rows past the
// projection read as zero, all issued before the dependency wait) and unpacks
// them chunk by chunk into int8 B tiles as they land.  It takes all its
// chunks of the tokens' codes (the quantiser's operand layout: NT rows of
// 128 B per chunk, chunks one after the other) with one bulk copy after the
// wait.  The A tile of chunk c is the 128-row window that starts at chunk c's
// codes: its rows past NT are whatever follows (later chunks, the B tiles),
// and they only reach TMEM lanes that are never read.  The int32 accumulator
// sits in TMEM (128 lanes = tokens, 256 columns = rows).  Each CTA stages its
// int32 sums in shared memory (over the B tiles, free once its MMAs are
// done); after a cluster barrier every CTA of the cluster forms y for its
// share of the slab's (token, 4-row group) items, adding the ksplit CTAs'
// sums through distributed shared memory, and a second cluster barrier keeps
// each CTA's sums in place until its peers have read them.  Nothing goes
// through global memory but the weights, the codes, the per-token values and
// y.
// Warp roles (16 warps):
//   warp 0      producer: weight chunks, then the codes
//   warp 1      TMEM allocation (256 columns); lane 0 issues the MMAs, with one
//               barrier wait and one commit per chunk
//   warp 2      per-token constants (code sums, dequantisation factors)
//   warps 8-15  unpack: thread = weight row, 2-bit codes -> int8 B tile
//   warps 0, 4, 8, 12 afterwards: tcgen05.ld of the token lanes (TMEM lanes
//               0 .. 31), 64 rows each, into shared memory
//   all         the cluster's reduction and y
// Every wait on an mbarrier is bounded; on timeout the CTA records the error,
// drains its copies and MMAs and frees TMEM.  Every CTA then still takes part
// in both cluster barriers (its peers wait there, unbounded), so a timeout
// ends the kernel with the error word set and the slab's y unspecified.
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kGwRows = 256;                 // weight rows per slab (MMA N)
constexpr int kGwThreads = 16 * 32;
constexpr int kGwUnpackThreads = 256;        // warps 8-15, one weight row each
constexpr int kGwSlots = 3;                  // unpacked weight chunks in flight (B tiles)
constexpr int kGwMaxProj = 8;
constexpr int kGwMaxChunksPerSplit = 32;     // 128-wide K chunks a CTA holds, at most
constexpr int kGwMaxCluster = 8;             // K ranges per slab: a portable cluster
constexpr int kGwAWindow = 128 * 128;        // bytes an A tile (128 rows x 128 B) spans from its start
constexpr int kGwBBytes = kGwRows * 128;     // B tile: 256 weight rows x 128 B
constexpr int kGwSmemBudget = 226 * 1024;    // dynamic shared memory, within the 227 KB a CTA may hold

struct GemvWideParams {
    const int8_t* codes;                      // per 128-wide K chunk, NT rows of 128 B (128-byte swizzled atoms)
    const float* absmax;                      // [M]   (fused mode)
    const int* qsum;                          // [M]
    const float* scale[kGwMaxProj];           // beta_g (fused mode)
    uint16_t* y[kGwMaxProj];                  // bf16 [M][N_g] (fused mode)
    int32_t* acc;                             // int32 [M][N]  (contraction-only mode, one projection)
    int rows[kGwMaxProj];                     // N_g
    int slab_start[kGwMaxProj + 1];           // prefix sums of ceil(N_g / 256)
    int nproj;
    int M, K;
    int ksplit;                               // K ranges per slab = the cluster size
    int chunks_per_split;                     // 128-wide K chunks per range
};

// The packed weights of each projection as a 2D tensor of uint32 words
// [N_g][K/16]; a copy is a box of 256 rows x 8 words (one 128-wide K chunk).
struct GemvWideMaps {
    CUtensorMap w[kGwMaxProj];
};

struct GemvWidePlan {
    int slabs, ksplit, chunks_per_split, grid;
    size_t smem_bytes;
};

// Shared memory: [codes: cps x NT x 128 B][3 B tiles][packed weights: 256
// rows x cps x 32 B]; the last chunk's A window reaches into the B tiles.
inline size_t gemv_wide_smem(int cps, int NT) {
    return static_cast<size_t>(cps) * NT * 128 + static_cast<size_t>(kGwSlots) * kGwBBytes +
           static_cast<size_t>(kGwRows) * cps * 32 + 1024;
}

// Cost of a launch in the model the plan minimises: per wave of clusters a
// fixed part (start, the first codes, the cluster's reduction and y) and a
// part per 128-wide K chunk a CTA holds (the MMA thread's issue sequence),
// from globaltimer stamps of the kernel at the 2.7B decode shapes.
constexpr int kGwFixedNs = 3000;
constexpr int kGwChunkNs = 480;

// `slabs` slabs of 256 rows (the projections' own, summed); each slab's K
// range in ksplit <= 8 pieces (a cluster; no empty pieces, at most 32 chunks
// a piece, the piece's weights within shared memory).  clusters[k] = clusters
// of k CTAs of this kernel that fit on the GPU at once (k = 1 .. 8).  Takes
// the ksplit of least modelled time; false if no piece fits.
inline bool gemv_wide_plan(int K, int NT, int64_t slabs64, const int* clusters, GemvWidePlan* plan) {
    const int nchunks = K / 128;
    if (slabs64 < 1 || nchunks < 1 || slabs64 * kGwMaxCluster > INT32_MAX) return false;
    const int slabs = static_cast<int>(slabs64);
    int64_t best = -1;
    for (int ks = 1; ks <= kGwMaxCluster && ks <= nchunks; ++ks) {
        const int cps = (nchunks + ks - 1) / ks;
        if ((nchunks + cps - 1) / cps != ks) continue;  // a piece would be empty: the smaller ksplit covers it
        if (cps > kGwMaxChunksPerSplit || gemv_wide_smem(cps, NT) > static_cast<size_t>(kGwSmemBudget)) continue;
        if (clusters[ks] < 1) continue;
        const int64_t waves = (slabs64 + clusters[ks] - 1) / clusters[ks];
        const int64_t t = waves * (kGwFixedNs + static_cast<int64_t>(cps) * kGwChunkNs);
        if (best < 0 || t < best) {
            best = t;
            plan->ksplit = ks;
            plan->chunks_per_split = cps;
        }
    }
    if (best < 0) return false;
    plan->slabs = slabs;
    plan->grid = slabs * plan->ksplit;
    plan->smem_bytes = gemv_wide_smem(plan->chunks_per_split, NT);
    return true;
}

// cluster barrier over all threads of the cluster's CTAs (release / acquire),
// whole or as its two halves
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_sync_all() {
    cluster_arrive();
    cluster_wait();
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// the address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t dsmem_addr(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

__device__ __forceinline__ int4 ld_dsmem_s32x4(uint32_t addr) {
    int4 v;
    asm volatile("ld.shared::cluster.v4.s32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

constexpr int kGwSumStride = kGwRows + 4;  // int32 words per token row of the staged sums (conflict-free)

template <int NT, bool FUSED>
__global__ void __launch_bounds__(kGwThreads, 1)
    gemv_wide_kernel(const __grid_constant__ GemvWideParams p, const __grid_constant__ GemvWideMaps maps) {
    static_assert(NT == 16 || NT == 32, "token rows of the codes: 16 or 32");
    static_assert(NT * kGwSumStride * 4 <= kGwSlots * kGwBBytes, "the staged sums fit the B slots");
    static_assert(kGwAWindow - NT * 128 <= kGwSlots * kGwBBytes, "the last A window stays within the B tiles");
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t w_bar[kGwMaxChunksPerSplit];
    __shared__ __align__(8) uint64_t codes_bar;            // all of the CTA's codes have landed
    __shared__ __align__(8) uint64_t ready[kGwSlots];      // B tile of the slot unpacked (unpack warps)
    __shared__ __align__(8) uint64_t slot_free[kGwSlots];  // the slot's MMAs are done (one commit)
    __shared__ __align__(8) uint64_t d_full;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_flag, w_issued, codes_issued;
    __shared__ int qs_s[NT];
    __shared__ float cm_s[NT];

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int cps = p.chunks_per_split;
    uint8_t* codes_s = smem;                                   // chunk c: NT x 128 B at codes_s + c * NT * 128
    uint8_t* b_base = smem + static_cast<size_t>(cps) * NT * 128;  // also, once the MMAs are done, the staged sums
    uint8_t* w_s = b_base + kGwSlots * kGwBBytes;              // chunk c: 256 rows x 32 B at w_s + c * 8 KB

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nchunks = p.K >> 7;
    const int ks = p.ksplit;
    const int slab = blockIdx.x / ks, kr = blockIdx.x % ks;
    int g = 0;  // projection of the slab
#pragma unroll
    for (int i = 1; i < kGwMaxProj; ++i)
        if (i < p.nproj && slab >= p.slab_start[i]) g = i;
    const int Ng = p.rows[g];
    const int n0 = (slab - p.slab_start[g]) * kGwRows;  // the slab's first row in projection g
    const int nrows = min(Ng - n0, kGwRows);
    const int c_lo = kr * cps;
    const int nch = min(cps, nchunks - c_lo);
    if (nrows <= 0 || nch <= 0) {  // the plan makes none; still meet the peers at both cluster barriers
        cluster_sync_all();
        cluster_sync_all();
        return;
    }

    if (threadIdx.x == 0) {
        for (int c = 0; c < nch; ++c) mbar_init(&w_bar[c], 1);
        mbar_init(&codes_bar, 1);
        for (int s = 0; s < kGwSlots; ++s) {
            mbar_init(&ready[s], kGwUnpackThreads / 32);  // one arrival per unpack warp
            mbar_init(&slot_free[s], 1);
        }
        mbar_init(&d_full, 1);
        abort_flag = 0;
        w_issued = 0;
        codes_issued = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_s, kGwRows);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            // the slab's packed weights for this K range are parameters: fetched
            // before the dependency wait, a box of 256 rows x 8 words per chunk
            // (rows past the projection are zero-filled and counted)
            prefetch_tensormap(&maps.w[g]);
            for (int c = 0; c < nch; ++c) {
                mbar_arrive_expect_tx(&w_bar[c], kGwRows * 32);
                tma_load_2d(w_s + c * (kGwRows * 32), &maps.w[g], (c_lo + c) * 8, n0, &w_bar[c]);
            }
            w_issued = nch;
            // the codes come from the kernel launched just before
            pdl_wait();
            pdl_launch_dependents();
            // the range's chunks are consecutive in the codes: one copy
            mbar_arrive_expect_tx(&codes_bar, static_cast<uint32_t>(nch) * NT * 128);
            bulk_g2s(codes_s, p.codes + static_cast<size_t>(c_lo) * NT * 128, static_cast<uint32_t>(nch) * NT * 128,
                     &codes_bar);
            codes_issued = 1;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(128, kGwRows);
            bool issued = false;
            const bool got_codes = mbar_wait(&codes_bar, 0, &abort_flag);
            for (int c = 0; c < nch && got_codes; ++c) {
                // one wait per chunk: the unpack warps' signal for its B tile
                const int s = c % kGwSlots;
                if (!mbar_wait(&ready[s], (c / kGwSlots) & 1, &abort_flag)) break;
                tc_fence_after();
                const uint32_t a0 = smem_u32(codes_s + c * NT * 128), b0 = smem_u32(b_base + s * kGwBBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_i8(tmem_base, sw128_kmajor_desc(a0 + 32 * kk), sw128_kmajor_desc(b0 + 32 * kk), idesc,
                           (c | kk) != 0 ? 1u : 0u);
                issued = true;
                mma_commit(&slot_free[s]);
            }
            if (issued) mma_commit(&d_full);
            if (issued && abort_flag) {  // d_full may never be waited on: let the MMAs drain here
                int zero = 0;
                mbar_wait(&d_full, 0, &zero);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ per-token constants
        pdl_wait();  // written by the kernel launched just before
        if (lane < p.M) {
            qs_s[lane] = p.qsum[lane];
            if constexpr (FUSED) cm_s[lane] = __fmul_rn(__fdiv_rn(p.absmax[lane], 127.0f), __ldg(p.scale[g]));
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ unpack
        const int r = threadIdx.x - 8 * 32;  // weight row of the slab, 0 .. 255 (past nrows: zeros)
        uint8_t* brow0 = b_base + (r >> 3) * 1024 + (r & 7) * 128;
        for (int c = 0; c < nch; ++c) {
            const int sb = c % kGwSlots;
            bool ok = mbar_wait(&w_bar[c], 0, &abort_flag);
            if (c >= kGwSlots) ok = ok && mbar_wait(&slot_free[sb], ((c / kGwSlots) - 1) & 1, &abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;
            const uint4* src = reinterpret_cast<const uint4*>(w_s + c * (kGwRows * 32) + r * 32);
            const uint4 pa = src[0], pb = src[1];
            const uint32_t words[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
            uint8_t* brow = brow0 + sb * kGwBBytes;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                // word t: K bytes 16t .. 16t + 15 of the chunk; byte-lane j of the
                // 16-byte unit gets codes 4j .. 4j + 3 (bits 2j of each byte)
                const uint32_t w = words[t];
                *reinterpret_cast<uint4*>(brow + ((t ^ (r & 7)) << 4)) =
                    make_uint4(w & 0x03030303u, (w >> 2) & 0x03030303u, (w >> 4) & 0x03030303u,
                               (w >> 6) & 0x03030303u);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ready[sb]);
        }
    }

    // warps 0, 4, 8, 12 reach TMEM lanes 0 .. 31 (lane = token): once the MMAs
    // are done (each waits itself), two blocks of 32 rows each into shared
    // memory over the B slots
    if ((warp & 3) == 0) {
        const bool got = mbar_wait(&d_full, 0, &abort_flag);
        if (__all_sync(0xffffffffu, got)) {  // tcgen05.ld wants the whole warp
            tc_fence_after();
            const int j0 = (warp >> 2) * 2;
            uint32_t v0[32], v1[32];
            tmem_ld_32x32b_x32(tmem_base + 32 * j0, v0);
            tmem_ld_32x32b_x32(tmem_base + 32 * (j0 + 1), v1);
            tmem_ld_wait();
            if (lane < NT) {
                uint32_t* srow = reinterpret_cast<uint32_t*>(b_base) + lane * kGwSumStride + 32 * j0;
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    *reinterpret_cast<uint4*>(srow + i) = make_uint4(v0[i], v0[i + 1], v0[i + 2], v0[i + 3]);
                    *reinterpret_cast<uint4*>(srow + 32 + i) = make_uint4(v1[i], v1[i + 1], v1[i + 2], v1[i + 3]);
                }
            }
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kGwRows);
    }
    if (abort_flag && threadIdx.x == 0) {
        // a wait gave up: every copy issued lands before the CTA can exit (the
        // error word is set; the slab's y is unspecified)
        int zero = 0;
        for (int c = 0; c < w_issued; ++c) mbar_wait(&w_bar[c], 0, &zero);
        if (codes_issued) mbar_wait(&codes_bar, 0, &zero);
    }
    // every CTA of the cluster has its sums staged
    cluster_sync_all();
    // this CTA's share of the slab's items (item i: token i / 64, rows
    // 4 (i % 64) .. + 3): the ks CTAs' sums added through distributed shared
    // memory, all of an item's loads in flight together
    const int items = p.M * (kGwRows / 4);
    const int per = (items + ks - 1) / ks;
    const int rank = static_cast<int>(cluster_rank());
    const int hi = min((rank + 1) * per, items);
    const uint32_t sums = smem_u32(b_base);
    for (int it = rank * per + static_cast<int>(threadIdx.x); it < hi; it += kGwThreads) {
        const int t = it >> 6, r = (it & 63) * 4;
        if (r >= nrows) continue;
        const uint32_t a = sums + static_cast<uint32_t>(t * kGwSumStride + r) * 4u;
        int4 part[kGwMaxCluster];
#pragma unroll
        for (int q = 0; q < kGwMaxCluster; ++q)
            if (q < ks) part[q] = ld_dsmem_s32x4(dsmem_addr(a, static_cast<uint32_t>(q)));
        const int qs = qs_s[t];
        int v[4] = {-qs, -qs, -qs, -qs};  // sum over K of c q, minus sum q: exact integers
#pragma unroll
        for (int q = 0; q < kGwMaxCluster; ++q)
            if (q < ks) {
                v[0] += part[q].x;
                v[1] += part[q].y;
                v[2] += part[q].z;
                v[3] += part[q].w;
            }
        const int cnt = min(4, nrows - r);
        const size_t o = static_cast<size_t>(t) * Ng + n0 + r;
        if constexpr (FUSED) {
            const float cm = cm_s[t];
            uint16_t yb[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                yb[j] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(static_cast<float>(v[j]), cm)));
            uint16_t* yo = p.y[g] + o;
            if (cnt == 4 && (reinterpret_cast<uintptr_t>(yo) & 7) == 0) {
                *reinterpret_cast<uint2*>(yo) = make_uint2(yb[0] | (static_cast<uint32_t>(yb[1]) << 16),
                                                           yb[2] | (static_cast<uint32_t>(yb[3]) << 16));
            } else {
                for (int j = 0; j < cnt; ++j) yo[j] = yb[j];
            }
        } else {
            int32_t* ao = p.acc + o;
            if (cnt == 4 && (reinterpret_cast<uintptr_t>(ao) & 15) == 0) {
                *reinterpret_cast<int4*>(ao) = make_int4(v[0], v[1], v[2], v[3]);
            } else {
                for (int j = 0; j < cnt; ++j) ao[j] = v[j];
            }
        }
    }
    // no CTA leaves while a peer may still read its sums
    cluster_sync_all();
}

}  // namespace mmf
