// chain.cuh -- a chain of small-M fused BitLinear calls (1 .. 3 tokens) in one
// persistent launch.
//
// At decode sizes one call moves a few MB of packed weights, under a
// microsecond of HBM time, while a launch of its own pays several
// microseconds of fixed cost: the dependency on the kernel before it, the
// copy of x, the normalisation's barriers, the tail of its CTAs. A model's
// decode step is a sequence of such calls, each reading what earlier ones
// wrote. This kernel runs the whole sequence with one CTA per SM, with the
// same arithmetic as the small-M decode kernel (RMSNorm, per-token absmax int8
// codes, the ternary add/sub rule of ld246.com section "三值权重的应用" on
// 2-bit codes by LOP3 + DP4A, the rescale by a/127 * beta), and two changes:
//   - Weights are parameters, so the producer warp streams each CTA's rows of
//     call after call into a ring of shared-memory slots, bounded only by free
//     slots: a call's weights arrive while earlier calls still compute.
//   - A call reads its input only after every CTA has finished the call
//     before: each CTA adds one to a counter in global memory when its rows of
//     a call are written, and a CTA starts call c once the counter reaches
//     c x (number of CTAs). So the results are those of launching the calls one
//     after another on a stream, and a call's x may be an earlier call's y.
//
// CTA: kChainWarps compute warps + 1 producer warp. Call c's rows (the
// concatenated row space of its projections) are split in contiguous slabs of
// rows_per_cta (a multiple of 4) over the CTAs; a slab is cut into stages of
// rows_per_stage rows, one ring slot each. The compute warps normalise and
// quantise the M tokens redundantly in every CTA (x in registers, fp64 sum of
// squares, three barriers), then take 4-row items round-robin: 8 lanes per
// row, a row's 8 partials meet in a warp-shuffle tree.
//
// Every wait is bounded. A spin that runs out records the timeout in the device
// error word and sets the CTA's abort flag; the compute warps agree on it at
// their next barrier and leave, the producer drains its copies and leaves, and
// the other CTAs' waits on the counter run out in turn. The launch is
// cooperative, so all CTAs are resident together (the launch fails otherwise).
#pragma once
#include "common.cuh"
#include "gemv.cuh"

namespace mmf {

constexpr int kChainWarps = 8;                               // compute warps
constexpr int kChainThreads = (kChainWarps + 1) * 32;
constexpr int kChainMaxTokens = 3;
constexpr int kChainMaxK = 8192;                             // x is held in registers
constexpr int kChainCpt = kChainMaxK / 8 / (kChainWarps * 32);  // 8-element chunks per thread
constexpr int kChainSlotBytes = 32768;
constexpr int kChainMaxSlots = 8;
constexpr int kChainSmemBudget = 220 * 1024;
constexpr int kChainBarrier = 1;                             // named barrier of the compute warps
constexpr int kChainCounterBytes = 256;                      // the counter's line, ahead of the calls

// One call of a chain in device memory, written by the host encoder.
struct ChainCall {
    const uint16_t* x;        // bf16 [M][K]; the gate g in GLU form
    const uint16_t* u;        // bf16 [M][K] in GLU form (p = bf16(SiLU(g) * u) is normalised), else null
    const float* gamma;       // fp32 [K]
    const uint32_t* packed[kGemvMaxProj];
    const float* scale[kGemvMaxProj];
    uint16_t* y[kGemvMaxProj];
    int row_start[kGemvMaxProj + 1];  // prefix sums of N_g
    float eps;
    int K;
    int nproj;
    int rows_per_cta;         // multiple of 4
    int rows_per_stage;       // multiple of 4; rows_per_stage * K/4 <= slot bytes
};

struct ChainParams {
    const ChainCall* calls;
    unsigned* counter;        // zeroed before the launch
    int ncalls;
    int M;
    int slots;                // ring slots of kChainSlotBytes
    int q_bytes;              // shared memory for the codes: M * (largest K), rounded up to 128
};

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Waits until *ctr >= target; false on abort or after kWaitLimitNs (then the
// timeout is recorded and the abort flag set).
__device__ __forceinline__ bool chain_wait(const unsigned* ctr, unsigned target, volatile int* abort_flag) {
    if (ld_acquire_gpu(ctr) >= target) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (;;) {
        if (ld_acquire_gpu(ctr) >= target) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_error_word, kErrTimeout);
            *abort_flag = 1;
            return false;
        }
    }
}

// Asynchronous global -> shared copies (LDGSTS) of parameters one call ahead.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// waits until at most n of this thread's committed groups are still in flight
template <int n>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(n) : "memory"); }

__device__ __forceinline__ void chain_sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(kChainBarrier), "n"(kChainWarps * 32) : "memory");
}

template <int MT>
__global__ void __launch_bounds__(kChainThreads, 1) gemv_chain_kernel(const __grid_constant__ ChainParams p) {
    constexpr int NW = kChainWarps;
    constexpr int NT = NW * 32;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t full_bar[kChainMaxSlots];
    __shared__ __align__(8) uint64_t empty_bar[kChainMaxSlots];
    __shared__ __align__(16) ChainCall desc_s[2];     // the compute warps' copy of call c's descriptor, in [c & 1]
    __shared__ __align__(16) ChainCall prod_desc[2];  // the producer warp's
    __shared__ float beta_s[2][kGemvMaxProj];
    __shared__ double red_d[NW][MT];
    __shared__ float red_f[NW][MT];
    __shared__ int red_i[NW][MT];
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.slots;
    const int G = gridDim.x;
    uint8_t* ring = smem;
    int8_t* q_s = reinterpret_cast<int8_t*>(smem + static_cast<size_t>(S) * kChainSlotBytes);
    float* gamma_s = reinterpret_cast<float*>(smem + static_cast<size_t>(S) * kChainSlotBytes + p.q_bytes);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], NW);
        }
        abort_flag = 0;
        mbar_fence_init();
    }
    __syncthreads();

    constexpr int kDescChunks = static_cast<int>(sizeof(ChainCall) / 16);
    static_assert(sizeof(ChainCall) % 16 == 0, "descriptor copied in 16-byte pieces");
    // call c's descriptor into buf[c & 1] by lanes 0 .. kDescChunks - 1, one copy group
    auto fetch_desc = [&](ChainCall* buf, int c) {
        if (lane < kDescChunks)
            cp_async16(reinterpret_cast<uint8_t*>(&buf[c & 1]) + 16 * lane,
                       reinterpret_cast<const uint8_t*>(p.calls + c) + 16 * lane);
        cp_async_commit();
    };

    if (warp == NW) {
        // ---------------- producer: this CTA's weight rows, call after call. The
        // warp copies each call's descriptor one call ahead; lane 0 brings the
        // call's x (and u) into L2 for the normalisation to come (L2 stays
        // coherent with writes that land later) and issues its weight stages.
        int g = 0;  // slot uses so far
        bool ok = true;
        fetch_desc(prod_desc, 0);
        for (int c = 0; c < p.ncalls && ok; ++c) {
            if (c + 1 < p.ncalls) {
                fetch_desc(prod_desc, c + 1);
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            __syncwarp();
            const ChainCall& cc = prod_desc[c & 1];
            if (lane == 0) {
                const int nproj = cc.nproj;
                const int R = cc.row_start[nproj];
                const int rowbytes = cc.K >> 2;
                const int rpc = cc.rows_per_cta, rps = cc.rows_per_stage;
                const int row0 = blockIdx.x * rpc;
                const int nrows = min(R - row0, rpc);
                if (nrows > 0) {
                    const uint32_t xb = static_cast<uint32_t>(2 * p.M * cc.K);
                    for (uint32_t off = 0; off < xb; off += 65536u) {
                        const uint32_t n = xb - off < 65536u ? xb - off : 65536u;
                        bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(cc.x) + off, n);
                        if (cc.u) bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(cc.u) + off, n);
                    }
                }
                for (int s = 0; s * rps < nrows; ++s, ++g) {
                    const int slot = g % S;
                    if (g >= S && !mbar_wait(&empty_bar[slot], ((g / S) - 1) & 1, &abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int r0 = row0 + s * rps;
                    const int r1 = min(r0 + rps, row0 + nrows);
                    mbar_arrive_expect_tx(&full_bar[slot], static_cast<uint32_t>(r1 - r0) * rowbytes);
                    uint8_t* dst = ring + static_cast<size_t>(slot) * kChainSlotBytes;
                    for (int r = r0; r < r1;) {  // split at projection boundaries
                        int gi = 0;
                        for (int i = 1; i < nproj; ++i)
                            if (r >= cc.row_start[i]) gi = i;
                        const int e = min(r1, cc.row_start[gi + 1]);
                        const uint8_t* src = reinterpret_cast<const uint8_t*>(cc.packed[gi]) +
                                             static_cast<size_t>(r - cc.row_start[gi]) * rowbytes;
                        bulk_g2s(dst + static_cast<size_t>(r - r0) * rowbytes, src,
                                 static_cast<uint32_t>(e - r) * rowbytes, &full_bar[slot]);
                        r = e;
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            __syncwarp();  // lane 0 is done with buffer c & 1 before it is refilled
        }
        cp_async_wait<0>();
        // Let every copy this CTA started land before the CTA can exit.
        if (lane == 0) {
            int zero = 0;
            for (int u = max(0, g - S); u < g; ++u) mbar_wait(&full_bar[u % S], (u / S) & 1, &zero);
        }
        return;
    }

    // ---------------- compute warps
    const int tid = threadIdx.x;
    const int rsub = lane >> 3;  // row of a 4-row item
    const int l8 = lane & 7;     // lane within the row
    int g = 0;                   // slot uses so far (the producer's count)
    // Parameters arrive one call ahead: call c's descriptor is copied while call
    // c - 1 runs, its gamma and beta once call c - 1 has its codes. Call 0's here.
    auto fetch_params = [&](int c) {  // all compute threads; desc_s[c & 1] visible
        const ChainCall& dn = desc_s[c & 1];
        if (dn.row_start[dn.nproj] > 0) {
            for (int i = tid; i < (dn.K >> 2); i += NT) cp_async16(gamma_s + 4 * i, dn.gamma + 4 * i);
            if (tid < dn.nproj) cp_async4(&beta_s[c & 1][tid], dn.scale[tid]);
        }
        cp_async_commit();  // one copy group per thread
    };
    if (warp == 0) {
        fetch_desc(desc_s, 0);
        cp_async_wait<0>();
    }
    chain_sync();
    fetch_params(0);
    for (int c = 0; c < p.ncalls; ++c) {
        ChainCall& d = desc_s[c & 1];
        // the next call's descriptor (its buffer held call c - 1's, now done);
        // this call's gamma and beta (this thread's copies) have landed
        if (warp == 0 && c + 1 < p.ncalls) {
            fetch_desc(desc_s, c + 1);
            cp_async_wait<1>();  // all but the descriptor just issued
        } else {
            cp_async_wait<0>();
        }
        // every CTA has written its rows of the call before
        bool ok = true;
        if (c > 0 && tid == 0) ok = chain_wait(p.counter, static_cast<unsigned>(c) * static_cast<unsigned>(G), &abort_flag);
        if (!named_barrier_and<kChainBarrier, NT>(ok)) break;

        const int K = d.K;
        const int R = d.row_start[d.nproj];
        const int rowbytes = K >> 2;
        const int rps = d.rows_per_stage;
        const int row0 = blockIdx.x * d.rows_per_cta;
        const int nrows = min(R - row0, d.rows_per_cta);
        if (nrows > 0) {
            // ---- RMSNorm + int8 codes of the M tokens (every CTA the whole rows)
            const int C8 = K >> 3;
            uint4 xv[MT][kChainCpt];
            double s2[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                s2[m] = 0.0;
#pragma unroll
                for (int j = 0; j < kChainCpt; ++j) {
                    const int ch = tid + NT * j;
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (m < p.M && ch < C8) {
                        // L2 loads: x may have been written by another CTA during this launch
                        v = __ldcg(reinterpret_cast<const uint4*>(d.x + static_cast<size_t>(m) * K) + ch);
                        if (d.u) v = glu_gate8(v, __ldcg(reinterpret_cast<const uint4*>(d.u + static_cast<size_t>(m) * K) + ch));
                    }
                    xv[m][j] = v;
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                    double sq[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const double lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
                        sq[i] = lo * lo + hi * hi;
                    }
                    s2[m] += (sq[0] + sq[1]) + (sq[2] + sq[3]);  // exact sums: the order does not matter
                }
                s2[m] = warp_sum_f64(s2[m]);
                if (lane == 0) red_d[warp][m] = s2[m];
            }
            chain_sync();
            float inv[MT], amax[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                double t[NW];
#pragma unroll
                for (int w = 0; w < NW; ++w) t[w] = red_d[w][m];
                const float ms = static_cast<float>(tree_sum<NW>(t) / static_cast<double>(K));
                inv[m] = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, d.eps)));
                amax[m] = 0.0f;
            }
            const float4* g4 = reinterpret_cast<const float4*>(gamma_s);
#pragma unroll
            for (int j = 0; j < kChainCpt; ++j) {
                const int ch = tid + NT * j;
                if (ch >= C8) continue;
                const float4 ga = g4[2 * ch], gb = g4[2 * ch + 1];
                const float gm[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const uint32_t w[4] = {xv[m][j].x, xv[m][j].y, xv[m][j].z, xv[m][j].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        amax[m] = fmaxf(amax[m], fabsf(__fmul_rn(__fmul_rn(__uint_as_float(w[i] << 16), inv[m]), gm[2 * i])));
                        amax[m] = fmaxf(amax[m], fabsf(__fmul_rn(__fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv[m]),
                                                                 gm[2 * i + 1])));
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                amax[m] = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax[m])));  // >= 0
                if (lane == 0) red_f[warp][m] = amax[m];
            }
            chain_sync();
            float sc[MT], deq[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                float t[NW];
#pragma unroll
                for (int w = 0; w < NW; ++w) t[w] = red_f[w][m];
                const float a = fmaxf(tree_max<NW>(t), 1e-5f);
                sc[m] = __fdiv_rn(127.0f, a);
                deq[m] = __fdiv_rn(a, 127.0f);
            }
            // codes: r * s rounded to the nearest integer, ties to even, by adding
            // 1.5 * 2^23 (the code is the low byte); |r * s| <= 127 up to an ulp, so
            // the clamp of the definition never acts. Layout t-major: the 16 codes
            // k = 64c + 16t .. +15 of token m at m*K + 16*(t*C + c), C = K/64.
            const int C64 = K >> 6;
            int qs[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) qs[m] = 0;
#pragma unroll
            for (int j = 0; j < kChainCpt; ++j) {
                const int ch = tid + NT * j;
                if (ch >= C8) continue;
                const float4 ga = g4[2 * ch], gb = g4[2 * ch + 1];
                const float gm[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m >= p.M) continue;
                    const uint32_t w[4] = {xv[m][j].x, xv[m][j].y, xv[m][j].z, xv[m][j].w};
                    uint32_t cb[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float xf = (i & 1) ? __uint_as_float(w[i >> 1] & 0xFFFF0000u) : __uint_as_float(w[i >> 1] << 16);
                        cb[i] = __float_as_uint(
                            __fadd_rn(__fmul_rn(__fmul_rn(__fmul_rn(xf, inv[m]), gm[i]), sc[m]), 12582912.0f));
                    }
                    const uint32_t o0 = __byte_perm(__byte_perm(cb[0], cb[1], 0x0040), __byte_perm(cb[2], cb[3], 0x0040), 0x5410);
                    const uint32_t o1 = __byte_perm(__byte_perm(cb[4], cb[5], 0x0040), __byte_perm(cb[6], cb[7], 0x0040), 0x5410);
                    qs[m] = __dp4a(static_cast<int>(o0), 0x01010101, qs[m]);
                    qs[m] = __dp4a(static_cast<int>(o1), 0x01010101, qs[m]);
                    *reinterpret_cast<uint2*>(q_s + static_cast<size_t>(m) * K + 16 * (((ch & 7) >> 1) * C64 + (ch >> 3)) +
                                              8 * (ch & 1)) = make_uint2(o0, o1);
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                qs[m] = __reduce_add_sync(0xffffffffu, qs[m]);
                if (lane == 0) red_i[warp][m] = qs[m];
            }
            if (warp == 0) cp_async_wait<0>();  // the next call's descriptor
            chain_sync();  // codes, code sums, the next descriptor visible; gamma no longer read
            if (c + 1 < p.ncalls) fetch_params(c + 1);
            int qsum[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                int t[NW];
#pragma unroll
                for (int w = 0; w < NW; ++w) t[w] = red_i[w][m];
                qsum[m] = tree_sum<NW>(t);
            }

            // ---- contraction: 4-row items, item i of the slab to warp i % NW
            const int nst = (nrows + rps - 1) / rps;
            for (int s = 0; s < nst; ++s, ++g) {
                const int slot = g % S;
                if (ok) ok = mbar_wait(&full_bar[slot], (g / S) & 1, &abort_flag);
                if (ok) {
                    const int rs = min(rps, nrows - s * rps);
                    const int i0 = (s * rps) >> 2;           // first item of the stage
                    const int i1 = i0 + ((rs + 3) >> 2);
                    int first = i0 + ((warp - i0) % NW + NW) % NW;
                    const uint8_t* stage = ring + static_cast<size_t>(slot) * kChainSlotBytes;
                    for (int it = first; it < i1; it += NW) {
                        const int rl = 4 * (it - i0) + rsub;  // row within the stage
                        const bool valid = rl < rs;
                        const uint4* wp = reinterpret_cast<const uint4*>(stage + static_cast<size_t>(valid ? rl : 0) * rowbytes);
                        int a[MT][4][4];
#pragma unroll
                        for (int m = 0; m < MT; ++m)
#pragma unroll
                            for (int t = 0; t < 4; ++t)
#pragma unroll
                                for (int j = 0; j < 4; ++j) a[m][t][j] = 0;
#pragma unroll 2
                        for (int ch = l8; ch < C64; ch += 8) {
                            const uint4 wa = wp[ch];
                            const uint32_t da[4] = {wa.x, wa.y, wa.z, wa.w};
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                const uint32_t m0 = da[t] & 0x03030303u, m1 = da[t] & 0x0C0C0C0Cu;
                                const uint32_t m2 = da[t] & 0x30303030u, m3 = da[t] & 0xC0C0C0C0u;
#pragma unroll
                                for (int m = 0; m < MT; ++m) {
                                    const uint4 qv = *reinterpret_cast<const uint4*>(q_s + static_cast<size_t>(m) * K +
                                                                                     16 * (t * C64 + ch));
                                    a[m][t][0] = dp4a_us(m0, qv.x, a[m][t][0]);
                                    a[m][t][1] = dp4a_us(m1, qv.y, a[m][t][1]);
                                    a[m][t][2] = dp4a_us(m2, qv.z, a[m][t][2]);
                                    a[m][t][3] = dp4a_us(m3, qv.w, a[m][t][3]);
                                }
                            }
                        }
                        // the row's projection and its index there
                        const int r = row0 + s * rps + rl;
                        int gi = 0;
#pragma unroll
                        for (int i = 1; i < kGemvMaxProj; ++i)
                            if (i < d.nproj && r >= d.row_start[i]) gi = i;
                        const int n = r - d.row_start[gi];
                        const int Ng = d.row_start[gi + 1] - d.row_start[gi];
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            int acc[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j) acc[j] = (a[m][0][j] + a[m][1][j]) + (a[m][2][j] + a[m][3][j]);
                            int t = acc[0] + (acc[1] >> 2) + (acc[2] >> 4) + (acc[3] >> 6);
                            t += __shfl_xor_sync(0xffffffffu, t, 1);
                            t += __shfl_xor_sync(0xffffffffu, t, 2);
                            t += __shfl_xor_sync(0xffffffffu, t, 4);
                            if (valid && l8 == 0 && m < p.M) {
                                const float cm = __fmul_rn(deq[m], beta_s[c & 1][gi]);
                                const __nv_bfloat16 yb = __float2bfloat16_rn(__fmul_rn(static_cast<float>(t - qsum[m]), cm));
                                d.y[gi][static_cast<size_t>(m) * Ng + n] = __bfloat16_as_ushort(yb);
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty_bar[slot]);
            }
        } else {
            if (warp == 0) cp_async_wait<0>();  // the next call's descriptor
            chain_sync();
            if (c + 1 < p.ncalls) fetch_params(c + 1);
        }
        // this CTA's rows of call c are written: count it (stores ordered
        // before the add by the barrier and the fence)
        if (!named_barrier_and<kChainBarrier, NT>(ok)) break;
        if (tid == 0) {
            __threadfence();
            atomicAdd(p.counter, 1u);
        }
    }
}

}  // namespace mmf
