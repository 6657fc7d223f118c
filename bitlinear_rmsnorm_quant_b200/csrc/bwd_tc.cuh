// bwd_tc.cuh -- the two products of the straight-through backward on the
// 5th-generation tensor cores (tcgen05, kind::f16: bf16 operands, fp32
// accumulators in TMEM).
//
// With the quantisers passed through unchanged (ld246.com, section
// "训练与优化：新的策略": a surrogate gradient, the straight-through
// estimator), the gradients at the normalised activations and at the latent
// weights are plain products:
//   dr[m][k] = sum_n dy[m][n] w~[n][k]                  (beta applied later)
//   dW[n][k] = sum_m dy[m][n] (q[m][k] * (absmax[m] / 127))
// Both are written as D[k][c] = sum_j A[k][j] B[c][j] with the k axis (the
// activation width) as the MMA's 128-row A side and c (tokens for dr, output
// rows for dW) as its B side, so one kernel serves both:
//   dr: A = w~^T, unpacked by converter warps from the 2-bit codes (ternary
//       values are exact in bf16); B = dy, loaded by TMA in the 128-byte
//       swizzled K-major layout (dy rows are contiguous along n, the
//       contraction).
//   dW: A = x_q^T, converted from the int8 codes with each token's scale
//       absmax / 127 applied on the way in (one bf16 rounding per element);
//       B = dy^T, loaded by TMA as MN-major tiles (dy rows are contiguous
//       along n, the B side's own axis).
// The converted A tile is written in the MN-major 128-byte-swizzled layout:
// the packed codes hold 16 consecutive k of one n in a word, and q holds
// consecutive k of one token, so contiguous k is what the sources give.
//
// Tile: 128 k x 256 c, contraction in stages of 64 (128 bytes of bf16).
// Persistent, one CTA per SM, two TMEM accumulators (512 columns) so a
// tile's epilogue overlaps the next tile's MMAs.  Warp roles (512 threads):
//   warp 0      TMA producer: the B tile and the raw A source per stage
//   warp 1      TMEM allocation; lane 0 issues tcgen05.mma and the commits
//   warps 4-7   epilogue, one per TMEM sub-partition: tcgen05.ld, fp32
//               stores out[c][k] (32 lanes = 32 consecutive k = 128 bytes)
//   warps 8-15  converters: raw codes -> bf16 A tile
// Every wait is bounded; on timeout the CTA records the error, drains its
// copies and MMAs, frees TMEM and exits.
#pragma once
#include "common.cuh"

namespace mmf {

constexpr int kBwRows = 128;                  // k per tile (MMA M)
constexpr int kBwCols = 256;                  // tokens / output rows per tile (MMA N)
constexpr int kBwKs = 64;                     // contraction elements per stage (128 bytes of bf16)
constexpr int kBwStages = 4;
constexpr int kBwConvWarps = 8;
constexpr int kBwThreads = 16 * 32;
constexpr int kBwABytes = kBwRows * kBwKs * 2;        // 16 KB converted A
constexpr int kBwBBytes = kBwCols * kBwKs * 2;        // 32 KB B
constexpr int kBwMnBlock = 64 * 8 * 2 * 8;            // 8192: 64 MN elements x 64 K (8 atoms of 1024 B)

// raw A source per stage: packed codes 64 n x 128 k (32 bytes a row), or int8
// codes 64 tokens x 128 k (128 bytes a row)
template <int MODE>
struct BwLayout {
    static constexpr int raw_bytes = MODE == 0 ? kBwKs * (kBwRows / 4) : kBwKs * kBwRows;
    static constexpr int stage_bytes = kBwABytes + kBwBBytes + raw_bytes;
    static constexpr int smem_bytes = kBwStages * stage_bytes + 1024;  // + alignment slack
};

struct BwParams {
    float* out;            // fp32 [cols][K]: dr [M][K] or dW [N][K]
    const float* absmax;   // [M]  (dW: the tokens' scales)
    int K;                 // rows of D (the activation width), row stride of out
    int cols;              // M (dr) or N (dW)
    int contr;             // N (dr) or M (dW)
    int row_tiles;         // K / 128
    int num_tiles;         // row_tiles * ceil(cols / 256)
};

// Shared-memory matrix descriptor of an MN-major operand in 128-byte swizzled
// atoms (8 K-rows x 128 bytes = 64 bf16 along MN): atoms of consecutive
// 8-row K groups 1024 bytes apart (stride byte offset), 64-element MN blocks
// kBwMnBlock bytes apart (leading byte offset); version 1, layout 2.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(kBwMnBlock >> 4) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// Instruction descriptor for kind::f16 with bf16 A and B and an fp32 D:
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format (1 = bf16),
//   bit 15 A major (1 = MN), bit 16 B major (0 = K, 1 = MN), bits 17-22 N >> 3, bits 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
           (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Byte offset of A element (mn, j) (mn the 128-row axis, j the contraction
// index within the stage) in the MN-major swizzled tile, for the first of
// eight consecutive mn (one 16-byte chunk).
__device__ __forceinline__ uint32_t bw_a_chunk_offset(int mn, int j) {
    const int r = j & 7;
    return static_cast<uint32_t>((mn >> 6) * kBwMnBlock + (j >> 3) * 1024 + r * 128 + ((((mn & 63) >> 3) ^ r) << 4));
}

// Four ternary codes c = w~ + 1 in the bytes of x (each 0, 1 or 2) -> the bf16
// bits of w~ for codes 0,1 (lo) and 2,3 (hi).  A byte permute looks each code
// up in an 8-byte table: low bytes {0x80, 0x00, 0x80} and high bytes
// {0xBF, 0x00, 0x3F} give -1.0 (0xBF80), 0 and +1.0 (0x3F80); selector
// nibbles c, c + 4 per code come from one multiply-add.
__device__ __forceinline__ void ternary4_to_bf16(uint32_t x, uint32_t& lo, uint32_t& hi) {
    constexpr uint32_t t_lo = 0x00800080u, t_hi = 0x003F00BFu;
    lo = __byte_perm(t_lo, t_hi, x * 0x11u + 0x4040u);
    hi = __byte_perm(t_lo, t_hi, (x >> 16) * 0x11u + 0x4040u);
}

// Four int8 codes in the bytes of v, times s, each rounded to bf16:
// (float)q by the exponent trick (2^23 + (q + 128) has q + 128 in its low
// byte; subtracting 2^23 + 128 is exact), one fp32 product, round to bf16.
__device__ __forceinline__ void int8x4_scaled_to_bf16(uint32_t v, float s, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = v ^ 0x80808080u;
    float f[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        f[i] = __fmul_rn(__fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540u + i)), 8388736.0f), s);
    const __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(f[2], f[3]);
    lo = *reinterpret_cast<const uint32_t*>(&a);
    hi = *reinterpret_cast<const uint32_t*>(&b);
}

// MODE 0: dr (A from packed ternary codes, B = dy K-major)
// MODE 1: dW (A from int8 codes x absmax / 127, B = dy^T MN-major)
template <int MODE>
__global__ void __launch_bounds__(kBwThreads, 1)
    gemm_bwd_kernel(const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ CUtensorMap tmap_raw,
                    const BwParams p) {
    using L = BwLayout<MODE>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kBwStages];
    __shared__ __align__(8) uint64_t conv_bar[kBwStages];
    __shared__ __align__(8) uint64_t empty_bar[kBwStages];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_flag;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    auto a_tile = [&](int s) { return smem + s * L::stage_bytes; };
    auto b_tile = [&](int s) { return smem + s * L::stage_bytes + kBwABytes; };
    auto r_tile = [&](int s) { return smem + s * L::stage_bytes + kBwABytes + kBwBBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = (p.contr + kBwKs - 1) / kBwKs;
    const int G = gridDim.x;
    constexpr uint32_t kTmemCols = 2 * kBwCols;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kBwStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&conv_bar[s], kBwConvWarps * 32);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], 4);
        }
        mbar_init(&drain_bar, 1);
        abort_flag = 0;
        mbar_fence_init();
        prefetch_tensormap(&tmap_b);
        prefetch_tensormap(&tmap_raw);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_s, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int g = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += G) {
                const int k0 = (tile % p.row_tiles) * kBwRows;
                const int c0 = (tile / p.row_tiles) * kBwCols;
                for (int ks = 0; ks < nk; ++ks, ++g) {
                    const int s = g % kBwStages;
                    if (g >= kBwStages && !mbar_wait(&empty_bar[s], ((g / kBwStages) - 1) & 1, &abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full_bar[s], kBwBBytes + L::raw_bytes);
                    if constexpr (MODE == 0) {
                        // dy[c0 .. c0+255][n = 64 ks ..]: one box of 64 n x 256 tokens
                        tma_load_2d(b_tile(s), &tmap_b, ks * kBwKs, c0, &full_bar[s]);
                        // packed rows n = 64 ks .., bytes k0/4 .. k0/4 + 31
                        tma_load_2d(r_tile(s), &tmap_raw, k0 / 4, ks * kBwKs, &full_bar[s]);
                    } else {
                        // dy[m = 64 ks ..][c0 + 64 j ..]: four MN blocks of 64 n x 64 tokens
#pragma unroll
                        for (int j = 0; j < kBwCols / 64; ++j)
                            tma_load_2d(b_tile(s) + j * kBwMnBlock, &tmap_b, c0 + 64 * j, ks * kBwKs, &full_bar[s]);
                        // q rows m = 64 ks .., bytes k0 .. k0 + 127
                        tma_load_2d(r_tile(s), &tmap_raw, k0, ks * kBwKs, &full_bar[s]);
                    }
                }
            }
            int zero = 0;
            for (int u = max(0, g - kBwStages); u < g; ++u)
                mbar_wait(&full_bar[u % kBwStages], (u / kBwStages) & 1, &zero);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(kBwRows, kBwCols, true, MODE == 1);
            bool issued_any = false, ok = true;
            int g = 0, li = 0;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += G, ++li) {
                const int buf = li & 1;
                if (li >= 2 && !mbar_wait(&tempty_bar[buf], ((li >> 1) - 1) & 1, &abort_flag)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(buf * kBwCols);
                for (int ks = 0; ks < nk; ++ks, ++g) {
                    const int s = g % kBwStages;
                    const uint32_t par = (g / kBwStages) & 1;
                    if (!mbar_wait(&full_bar[s], par, &abort_flag) || !mbar_wait(&conv_bar[s], par, &abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(a_tile(s)), b0 = smem_u32(b_tile(s));
#pragma unroll
                    for (int kk = 0; kk < kBwKs / 16; ++kk) {
                        // 16 contraction elements = two 8-row K groups of the MN-major A (2048 bytes);
                        // 32 bytes along a K-major B row, 2048 bytes of an MN-major B
                        const uint64_t ad = sw128_mnmajor_desc(a0 + 2048 * kk);
                        const uint64_t bd = MODE == 0 ? sw128_kmajor_desc(b0 + 32 * kk) : sw128_mnmajor_desc(b0 + 2048 * kk);
                        mma_bf16(d, ad, bd, idesc, (ks | kk) != 0 ? 1u : 0u);
                    }
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
    } else if (warp >= 8) {
        // ------------------------------------------------------------ converters
        const int t = threadIdx.x - 8 * 32;  // 0 .. 255
        const int j = t >> 2;                // contraction row of the stage (n for dr, token for dW)
        const int part = t & 3;              // quarter of the 128 k
        int g = 0;
        bool ok = true;
        // dW: token j's absmax of stage ks depends on ks alone (every tile runs the same
        // contraction), so each thread loads it two stages ahead and the load's latency
        // stays off the conversion
        const auto absmax_at = [&](int ks) -> float {
            const int m = ks * kBwKs + j;
            return m < p.contr ? __ldg(p.absmax + m) : 0.0f;
        };
        float am_cur = 0.0f, am_next = 0.0f;
        if constexpr (MODE == 1) {
            am_cur = absmax_at(0);
            am_next = absmax_at(nk > 1 ? 1 : 0);
        }
        for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += G) {
            for (int ks = 0; ks < nk; ++ks, ++g) {
                const int s = g % kBwStages;
                float sc = 0.0f;
                if constexpr (MODE == 1) {
                    const float am_far = absmax_at((ks + 2) % nk);
                    sc = __fdiv_rn(am_cur, 127.0f);
                    am_cur = am_next;
                    am_next = am_far;
                }
                if (!mbar_wait(&full_bar[s], (g / kBwStages) & 1, &abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t* a = a_tile(s);
                if constexpr (MODE == 0) {
                    // row j: 8 words of 16 codes (k = 16 w .. 16 w + 15); this thread takes words 2 part, 2 part + 1
                    const uint2 wv = *reinterpret_cast<const uint2*>(r_tile(s) + j * 32 + 8 * part);
                    const uint32_t words[2] = {wv.x, wv.y};
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int kw = 16 * (2 * part + h);
                        uint32_t o[8];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            // codes of k = kw + 4q .. kw + 4q + 3 in the four bytes
                            ternary4_to_bf16((words[h] >> (2 * q)) & 0x03030303u, o[2 * q], o[2 * q + 1]);
                        }
                        *reinterpret_cast<uint4*>(a + bw_a_chunk_offset(kw, j)) = make_uint4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<uint4*>(a + bw_a_chunk_offset(kw + 8, j)) = make_uint4(o[4], o[5], o[6], o[7]);
                    }
                } else {
                    // token j: 128 int8 codes; this thread takes k = 32 part .. 32 part + 31, the
                    // two 16-byte halves in an order that alternates with j so the warp's reads
                    // spread over all eight 16-byte bank groups of the 128-byte rows
                    const uint4* src = reinterpret_cast<const uint4*>(r_tile(s) + j * 128 + 32 * part);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int h = hh ^ (j & 1);
                        const uint4 v = src[h];
                        const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
                        uint32_t o[8];
#pragma unroll
                        for (int q = 0; q < 4; ++q) int8x4_scaled_to_bf16(vw[q], sc, o[2 * q], o[2 * q + 1]);
                        const int kc = 32 * part + 16 * h;
                        *reinterpret_cast<uint4*>(a + bw_a_chunk_offset(kc, j)) = make_uint4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<uint4*>(a + bw_a_chunk_offset(kc + 8, j)) = make_uint4(o[4], o[5], o[6], o[7]);
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(&conv_bar[s]);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        const int wq = warp & 3;  // TMEM lanes 32 wq .. 32 wq + 31 = rows k0 + 32 wq ..
        int li = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += G, ++li) {
            const int buf = li & 1;
            const int k0 = (tile % p.row_tiles) * kBwRows;
            const int c0 = (tile / p.row_tiles) * kBwCols;
            const bool got = mbar_wait(&tfull_bar[buf], (li >> 1) & 1, &abort_flag);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            float* orow = p.out + k0 + 32 * wq + lane;
#pragma unroll 1
            for (int cc = 0; cc < kBwCols / 32; ++cc) {
                const int cb = c0 + 32 * cc;
                if (cb >= p.cols) break;  // uniform across the warp
                uint32_t r[32];
                const uint32_t taddr =
                    tmem_base + static_cast<uint32_t>(buf * kBwCols) + (static_cast<uint32_t>(32 * wq) << 16) + 32 * cc;
                tmem_ld_32x32b_x32(taddr, r);
                tmem_ld_wait();
                // column i of the chunk: the warp's 32 lanes store 32 consecutive k (128 bytes)
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (cb + i < p.cols) __stcs(orow + static_cast<size_t>(cb + i) * p.K, __uint_as_float(r[i]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty_bar[buf]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace mmf
