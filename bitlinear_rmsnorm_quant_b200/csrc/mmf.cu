// mmf.cu -- the C ABI of libmmf.so (declared in include/mmf.h): argument
// checks, kernel dispatch by M, tensor-map construction.  All kernels live in
// the headers included below; this is the only translation unit.
#include "mmf.h"

#include <cudaTypedefs.h>

#include <mutex>
#include <utility>

#include "common.cuh"
#include "copy.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "gemv_wide.cuh"
#include "pack.cuh"
#include "quant.cuh"
#include "scan.cuh"
#include "bwd.cuh"
#include "bwd_tc.cuh"

namespace {

using namespace mmf;

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;
constexpr int64_t kMaxK = 65536;  // the quantiser stages one bf16 row (2K bytes) in shared memory
constexpr int64_t kMaxTokens = int64_t(65535) * 256;  // tokens per call (16,776,960)

struct DeviceState {
    bool ready = false;
    int num_sms = 0;
    int wide_clusters[kGwMaxCluster + 1] = {};  // clusters of k decode tensor-core CTAs resident at once
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;

// Scratch of mmf_bitlinear_fwd_noalloc: the large-M workspace (int8 codes,
// absmax, per-token sums) lives here instead of in caller memory.  Every GPU
// that loads the library holds these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = MMF_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
// Device address of g_noalloc_scratch on each device (host code cannot use the
// symbol's name as an address); filled on the first call on that device.
void* g_noalloc_scratch_ptr[kMaxDevices];

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

template <typename F>
cudaError_t set_smem(F* f, size_t bytes) {
    return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

template <int BT>
cudaError_t set_tc_attrs() {
    cudaError_t e = set_smem(gemm_tc_kernel<BT, true>, TcLayout<BT>::smem_bytes);
    if (e == cudaSuccess) e = set_smem(gemm_tc_kernel<BT, false>, TcLayout<BT>::smem_bytes);
    return e;
}

template <int MT>
cudaError_t set_gemv_attrs() {
    cudaError_t e = set_smem(gemv_kernel<MT, true>, kGemvSmemBudget);
    if (e == cudaSuccess) e = set_smem(gemv_kernel<MT, false>, kGemvSmemBudget);
    if (e == cudaSuccess) e = set_smem(gemv_kernel<MT, true, true>, kGemvSmemBudget);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gemv_kernel<MT, true, true>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    // All of the SM's unified memory as shared memory: a CTA of the next kernel
    // can then join a running one without the SM first draining to change the
    // split between L1 and shared memory (these kernels stage everything they
    // read in shared memory).
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gemv_kernel<MT, true>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gemv_kernel<MT, false>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    return e;
}

// Per-device one-time set-up (device properties, kernel attributes, the driver
// entry point for tensor maps).  Must run before any stream capture.
mmf_status device_state(DeviceState** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MMF_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& st = g_dev[dev];
    if (!st.ready) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MMF_ERR_CUDA;
        if (prop.major != 10) return MMF_ERR_NO_DEVICE;
        st.num_sms = prop.multiProcessorCount;
        cudaError_t e = cudaSuccess;
        if (e == cudaSuccess) e = set_tc_attrs<16>();
        if (e == cudaSuccess) e = set_tc_attrs<32>();
        if (e == cudaSuccess) e = set_tc_attrs<64>();
        if (e == cudaSuccess) e = set_tc_attrs<128>();
        if (e == cudaSuccess) e = set_tc_attrs<256>();
        if (e == cudaSuccess) e = set_smem(gemv_wide_kernel<16, true>, kGwSmemBudget);
        if (e == cudaSuccess) e = set_smem(gemv_wide_kernel<16, false>, kGwSmemBudget);
        if (e == cudaSuccess) e = set_smem(gemv_wide_kernel<32, true>, kGwSmemBudget);
        if (e == cudaSuccess) e = set_smem(gemv_wide_kernel<32, false>, kGwSmemBudget);
        if (e == cudaSuccess) e = set_gemv_attrs<1>();
        if (e == cudaSuccess) e = set_gemv_attrs<2>();
        if (e == cudaSuccess) e = set_gemv_attrs<3>();
        if (e == cudaSuccess) e = set_smem(rmsnorm_quant_kernel<8>, 2 * kMaxK);  // one row of the largest K
        if (e == cudaSuccess) e = set_smem(rmsnorm_quant_kernel<8, true>, 2 * kMaxK);
        if (e == cudaSuccess) e = set_smem(gemm_bwd_kernel<0>, BwLayout<0>::smem_bytes);
        if (e == cudaSuccess) e = set_smem(gemm_bwd_kernel<1>, BwLayout<1>::smem_bytes);
        if (e == cudaSuccess) e = set_smem(mlgru_scan_tma_kernel, kStSmemBytes);
        if (e != cudaSuccess) return MMF_ERR_CUDA;
        // how many clusters of k CTAs of the decode tensor-core kernel (one CTA
        // per SM) the GPU holds at once: its plan keeps a launch to one wave
        for (int k = 1; k <= kGwMaxCluster; ++k) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(static_cast<unsigned>(k));
            cfg.blockDim = dim3(kGwThreads);
            cfg.dynamicSmemBytes = kGwSmemBudget;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = static_cast<unsigned>(k);
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, gemv_wide_kernel<32, true>, &cfg) != cudaSuccess) {
                (void)cudaGetLastError();
                n = k == 1 ? st.num_sms : 0;
            }
            st.wide_clusters[k] = n;
        }
        if (!g_encode_tiled) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || !fn)
                return MMF_ERR_CUDA;
            g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        st.ready = true;
    }
    *out = &st;
    return MMF_OK;
}

inline mmf_status launch_status() { return cudaGetLastError() == cudaSuccess ? MMF_OK : MMF_ERR_CUDA; }

mmf_status check_shape(int64_t M, int64_t K, int64_t N) {
    if (M < 0 || N < 0 || K < 0) return MMF_ERR_INVALID_ARG;
    if (K < 128 || (K % 128) != 0 || K > kMaxK) return MMF_ERR_UNSUPPORTED_SHAPE;
    if (M > kMaxDim || N > kMaxDim) return MMF_ERR_UNSUPPORTED_SHAPE;
    if (M > kMaxTokens) return MMF_ERR_UNSUPPORTED_SHAPE;  // the range the header states
    if (M * K > (int64_t(1) << 40) || N * K > (int64_t(1) << 40)) return MMF_ERR_UNSUPPORTED_SHAPE;
    return MMF_OK;
}

// Small M: up to kDecodeTcMinM - 1 tokens the CUDA-core decode kernel (its
// add/sub cost grows with M, about M/4 integer instructions per weight); from
// there to kDecodeTcMaxM the decode tensor-core kernel after a quantiser
// launch (its cost hardly depends on M: per CTA a fixed start and cluster
// reduction, and one MMA issue sequence per 128-wide K chunk); beyond, the
// large-M path.  Through a 2.7B layer set (4 calls, CUDA graph) the two decode
// kernels take 35 and 41 us at 3 tokens, 46 and 42 us at 4.
constexpr int64_t kDecodeTcMinM = 4;
constexpr int64_t kDecodeTcMaxM = 32;

bool takes_gemv(int64_t M, int64_t K) {
    if (M >= kDecodeTcMinM) return false;
    GemvPlan plan;
    return gemv_plan(static_cast<int>(M), static_cast<int>(K), 1, 148, &plan);
}

int decode_tc_nt(int64_t M) { return M <= 16 ? 16 : 32; }

bool takes_decode_tc(int64_t M, int64_t) { return M >= kDecodeTcMinM && M <= kDecodeTcMaxM; }

// Launches a kernel, as a programmatic dependent of the previous kernel on the
// stream when `pdl` is set.
template <typename... KArgs, typename... Args>
mmf_status launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                  Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
        (void)cudaGetLastError();
        return MMF_ERR_CUDA;
    }
    return MMF_OK;
}

// The same, in thread-block clusters of `cluster` CTAs along x.
template <typename... KArgs, typename... Args>
mmf_status launch_clustered(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                            int cluster, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
        (void)cudaGetLastError();
        return MMF_ERR_CUDA;
    }
    return MMF_OK;
}

int token_tile(int64_t M) {
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 256;
}

struct Workspace {
    int8_t* q;
    float* absmax;
    int* qsum;
};

size_t workspace_size_tc(int64_t M, int64_t K) {
    return align256(static_cast<size_t>(M) * K) + 2 * align256(4 * static_cast<size_t>(M));
}

// decode tensor-core path: the codes in the operand layout of NT rows, absmax, qsum
size_t workspace_size_dtc(int64_t M, int64_t K) {
    return align256(static_cast<size_t>(decode_tc_nt(M)) * K) + 2 * align256(4 * static_cast<size_t>(M));
}

Workspace carve_dtc(void* ws, int64_t M, int64_t K) {
    uint8_t* b = static_cast<uint8_t*>(ws);
    const size_t cb = align256(static_cast<size_t>(decode_tc_nt(M)) * K);
    Workspace w;
    w.q = reinterpret_cast<int8_t*>(b);
    w.absmax = reinterpret_cast<float*>(b + cb);
    w.qsum = reinterpret_cast<int*>(b + cb + align256(4 * static_cast<size_t>(M)));
    return w;
}

mmf_status encode_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t cols, int64_t rows,
                     int64_t pitch, int box_cols, int box_rows, CUtensorMapSwizzle swz);

// The projections (N > 0) of a decode tensor-core call.
struct WideGroup {
    int n = 0;
    const uint32_t* packed[kGwMaxProj];
    const float* scale[kGwMaxProj];
    uint16_t* y[kGwMaxProj];
    int64_t N[kGwMaxProj];
    int64_t slabs() const {
        int64_t s = 0;
        for (int g = 0; g < n; ++g) s += (N[g] + kGwRows - 1) / kGwRows;
        return s;
    }
};

// The decode tensor-core contraction of a group whose codes, absmax and qsum
// are in w (and whose partial sums and counters the quantiser has cleared).
mmf_status launch_gemv_wide(int NT, bool fused, const WideGroup& gr, const GemvWidePlan& plan, const Workspace& w,
                            int64_t M, int64_t K, int32_t* acc, cudaStream_t s) {
    GemvWideParams p{};
    GemvWideMaps maps{};
    p.codes = w.q;
    p.absmax = w.absmax;
    p.qsum = w.qsum;
    p.acc = acc;
    p.nproj = gr.n;
    p.M = static_cast<int>(M);
    p.K = static_cast<int>(K);
    p.ksplit = plan.ksplit;
    p.chunks_per_split = plan.chunks_per_split;
    p.slab_start[0] = 0;
    for (int g = 0; g < gr.n; ++g) {
        p.scale[g] = gr.scale[g];
        p.y[g] = gr.y[g];
        p.rows[g] = static_cast<int>(gr.N[g]);
        p.slab_start[g + 1] = p.slab_start[g] + static_cast<int>((gr.N[g] + kGwRows - 1) / kGwRows);
        // [N_g][K/16] words, boxes of 256 rows x one 128-wide K chunk (8 words)
        mmf_status st = encode_2d(&maps.w[g], CU_TENSOR_MAP_DATA_TYPE_UINT32, gr.packed[g], K / 16, gr.N[g], K / 4, 8,
                                  kGwRows, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (st != MMF_OK) return st;
    }
    // a programmatic dependent of the kernel launched just before it (which
    // wrote the codes): only the packed weights are read before the wait; a
    // cluster per slab, one CTA per K range
    const dim3 grid(static_cast<unsigned>(plan.grid)), block(kGwThreads);
    const int ks = plan.ksplit;
    if (NT == 16)
        return fused ? launch_clustered(gemv_wide_kernel<16, true>, grid, block, plan.smem_bytes, s, true, ks, p, maps)
                     : launch_clustered(gemv_wide_kernel<16, false>, grid, block, plan.smem_bytes, s, true, ks, p, maps);
    return fused ? launch_clustered(gemv_wide_kernel<32, true>, grid, block, plan.smem_bytes, s, true, ks, p, maps)
                 : launch_clustered(gemv_wide_kernel<32, false>, grid, block, plan.smem_bytes, s, true, ks, p, maps);
}

Workspace carve(void* ws, int64_t M, int64_t K) {
    uint8_t* b = static_cast<uint8_t*>(ws);
    Workspace w;
    w.q = reinterpret_cast<int8_t*>(b);
    w.absmax = reinterpret_cast<float*>(b + align256(static_cast<size_t>(M) * K));
    w.qsum = reinterpret_cast<int*>(b + align256(static_cast<size_t>(M) * K) + align256(4 * static_cast<size_t>(M)));
    return w;
}

mmf_status make_maps(const int8_t* q, const uint32_t* packed, int64_t M, int64_t K, int64_t N, int BT,
                     CUtensorMap* mq, CUtensorMap* mw) {
    const cuuint32_t es[2] = {1, 1};
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcK), static_cast<cuuint32_t>(BT)};
        if (g_encode_tiled(mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(q), dims, strides, box, es,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MMF_ERR_CUDA;
    }
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 4), static_cast<cuuint64_t>(N)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 4)};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcK / 4), static_cast<cuuint32_t>(kTcRows)};
        if (g_encode_tiled(mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint32_t*>(packed), dims, strides, box, es,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MMF_ERR_CUDA;
    }
    return MMF_OK;
}

// A 2D tensor map over a row-major [rows][cols] array of `esize`-byte elements
// with row pitch `pitch` bytes (a multiple of 16), box {box_cols, box_rows}.
mmf_status encode_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t cols, int64_t rows,
                     int64_t pitch, int box_cols, int box_rows, CUtensorMapSwizzle swz) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(pitch)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t es[2] = {1, 1};
    if (g_encode_tiled(map, dtype, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return MMF_ERR_CUDA;
    return MMF_OK;
}

template <int BT>
mmf_status launch_tc_bt(bool fused, const CUtensorMap& mq, const CUtensorMap& mw, TcParams p, cudaStream_t s,
                        bool pdl, int num_sms) {
    const int64_t tiles = ((static_cast<int64_t>(p.N) + kTcRows - 1) / kTcRows) *
                          ((static_cast<int64_t>(p.M) + BT - 1) / BT);
    if (tiles > kMaxDim) return MMF_ERR_UNSUPPORTED_SHAPE;
    p.n_tiles = (p.N + kTcRows - 1) / kTcRows;
    p.num_tiles = static_cast<int>(tiles);
    // the last, partial wave of R tiles as 2R half-token items when they fit
    // one wave (each CTA then spends half a tile there instead of a tile)
    p.full_items = p.num_tiles;
    p.num_items = p.num_tiles;
    if (BT == 256) {
        const int rem = p.num_tiles % num_sms;
        if (rem > 0 && 2 * rem <= num_sms) {
            p.full_items = p.num_tiles - rem;
            p.num_items = p.full_items + 2 * rem;
        }
    }
    const dim3 grid(static_cast<unsigned>(p.num_items < num_sms ? p.num_items : num_sms));  // persistent
    if (fused) return launch(gemm_tc_kernel<BT, true>, grid, dim3(kTcThreads), TcLayout<BT>::smem_bytes, s, pdl, mq, mw, p);
    return launch(gemm_tc_kernel<BT, false>, grid, dim3(kTcThreads), TcLayout<BT>::smem_bytes, s, pdl, mq, mw, p);
}

mmf_status launch_tc(bool fused, const int8_t* q, const uint32_t* packed, const TcParams& p, cudaStream_t s,
                     bool pdl, int num_sms) {
    const int BT = token_tile(p.M);
    CUtensorMap mq, mw;
    mmf_status st = make_maps(q, packed, p.M, p.K, p.N, BT, &mq, &mw);
    if (st != MMF_OK) return st;
    switch (BT) {
        case 16: return launch_tc_bt<16>(fused, mq, mw, p, s, pdl, num_sms);
        case 32: return launch_tc_bt<32>(fused, mq, mw, p, s, pdl, num_sms);
        case 64: return launch_tc_bt<64>(fused, mq, mw, p, s, pdl, num_sms);
        case 128: return launch_tc_bt<128>(fused, mq, mw, p, s, pdl, num_sms);
        default: return launch_tc_bt<256>(fused, mq, mw, p, s, pdl, num_sms);
    }
}

template <bool FUSED, bool GLU = false>
mmf_status launch_gemv(const GemvParams& p, const GemvPlan& plan, cudaStream_t s, bool pdl) {
    const dim3 grid(static_cast<unsigned>(plan.grid));
    switch (p.M) {
#define MMF_GEMV_CASE(MT) \
    case MT: return launch(gemv_kernel<MT, FUSED, GLU>, grid, dim3(gemv_threads(MT)), plan.smem_bytes, s, pdl, p);
        MMF_GEMV_CASE(1)
        MMF_GEMV_CASE(2)
        MMF_GEMV_CASE(3)
#undef MMF_GEMV_CASE
        default: return MMF_ERR_UNSUPPORTED_SHAPE;
    }
}


mmf_status launch_quant(const uint16_t* x, const float* gamma, float eps, int64_t M, int64_t K, int8_t* q,
                        float* absmax, int* qsum, cudaStream_t s, bool pdl, int num_sms,
                        const uint16_t* u = nullptr, int bl_nt = 0) {
    const dim3 rows_grid(static_cast<unsigned>(bl_nt > 0 ? bl_nt : M));
    if (u)  // GLU: one CTA of 8 warps per row, forming SiLU(g) * u on the way
        return launch(rmsnorm_quant_kernel<8, true>, rows_grid, dim3(256), static_cast<size_t>(K) * 2, s, pdl, x,
                      gamma, eps, static_cast<int>(K), M, q, absmax, qsum, u, bl_nt);
    if (bl_nt > 0 || M < kQuantWarpRowMinM || K > kMaxQuantRegK)  // one CTA of 8 warps per row
        return launch(rmsnorm_quant_kernel<8>, rows_grid, dim3(256), static_cast<size_t>(K) * 2, s, pdl, x, gamma, eps,
                      static_cast<int>(K), M, q, absmax, qsum, static_cast<const uint16_t*>(nullptr), bl_nt);
    // persistent: rows in registers, WPR warps per row (K <= 2048 WPR), as many
    // CTAs as fit on the SMs at once, never more than the rows need; up to
    // K = 6912, three warps of 9 chunks a lane rather than four of 7 (3.6%
    // faster at 8192 x 6912)
    int wpr = static_cast<int>((K + 2047) / 2048);
    if (wpr == 4 && K <= 3 * 32 * 9 * 8) wpr = 3;
    // 16-byte chunks a lane holds: as few as the width needs (fewer registers
    // for the row and its successor in flight)
    const int ch = static_cast<int>((K / 8 + 32 * wpr - 1) / (32 * wpr));
    using QuantRegFn = void (*)(const uint16_t*, const float*, float, int, int64_t, int8_t*, float*, int*);
    QuantRegFn kern;
    switch (wpr) {
        case 1: kern = ch <= 4 ? rmsnorm_quant_reg_kernel<1, 4> : ch <= 6 ? rmsnorm_quant_reg_kernel<1, 6>
                                                                          : rmsnorm_quant_reg_kernel<1, 8>; break;
        case 2: kern = ch <= 5 ? rmsnorm_quant_reg_kernel<2, 5> : ch <= 6 ? rmsnorm_quant_reg_kernel<2, 6>
                                                                          : rmsnorm_quant_reg_kernel<2, 8>; break;
        case 3: kern = ch <= 8 ? rmsnorm_quant_reg_kernel<3, 8> : rmsnorm_quant_reg_kernel<3, 9>; break;
        default: kern = ch <= 7 ? rmsnorm_quant_reg_kernel<4, 7> : rmsnorm_quant_reg_kernel<4, 8>; break;
    }
    const int threads = quant_reg_warps(wpr) * 32;
    const int rpc = quant_reg_warps(wpr) / wpr;
    const size_t smem = static_cast<size_t>(K) * 4;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess || per_sm < 1)
        return MMF_ERR_CUDA;
    int64_t grid = static_cast<int64_t>(per_sm) * num_sms;
    const int64_t need = (M + rpc - 1) / rpc;
    if (grid > need) grid = need;
    return launch(kern, dim3(static_cast<unsigned>(grid)), dim3(threads), smem, s, pdl, x, gamma, eps,
                  static_cast<int>(K), M, q, absmax, qsum);
}

// The fused forward of `count` projections that share x.  Arguments checked.
// u != null: GLU mode, x is the gate g and p = bf16(SiLU(g) * u) is the input.
mmf_status fwd_impl(const uint16_t* x, const float* gamma, float eps, int64_t M, int64_t K,
                    const mmf_projection* proj, int count, void* workspace, unsigned flags, cudaStream_t s,
                    DeviceState* dev, const uint16_t* u = nullptr) {
    const bool pdl = (flags & MMF_FWD_PDL) != 0;
    int64_t R = 0;
    for (int i = 0; i < count; ++i) R += proj[i].N;
    if (R == 0) return MMF_OK;
    GemvPlan plan;
    if (M < kDecodeTcMinM && gemv_plan(static_cast<int>(M), static_cast<int>(K), R, dev->num_sms, &plan)) {
        GemvParams p{};
        p.x = x;
        p.u = u;
        p.gamma = gamma;
        p.eps = eps;
        p.M = static_cast<int>(M);
        p.K = static_cast<int>(K);
        int g = 0;
        p.row_start[0] = 0;
        for (int i = 0; i < count; ++i) {
            if (proj[i].N == 0) continue;
            p.packed[g] = proj[i].packed;
            p.scale[g] = proj[i].scale;
            p.y[g] = proj[i].y;
            p.row_start[g + 1] = p.row_start[g] + static_cast<int>(proj[i].N);
            ++g;
        }
        p.nproj = g;
        p.rows_per_stage = plan.rows_per_stage;
        p.rows_per_cta = plan.rows_per_cta;
        p.stage_bytes = plan.stage_bytes;
        p.stages = plan.stages;
        return u ? launch_gemv<true, true>(p, plan, s, pdl) : launch_gemv<true>(p, plan, s, pdl);
    }
    if (takes_decode_tc(M, K)) {
        const int NT = decode_tc_nt(M);
        WideGroup gr;
        for (int i = 0; i < count; ++i) {
            if (proj[i].N == 0) continue;
            gr.packed[gr.n] = proj[i].packed;
            gr.scale[gr.n] = proj[i].scale;
            gr.y[gr.n] = proj[i].y;
            gr.N[gr.n] = proj[i].N;
            ++gr.n;
        }
        GemvWidePlan wplan;
        if (!gemv_wide_plan(static_cast<int>(K), NT, gr.slabs(), dev->wide_clusters, &wplan)) return MMF_ERR_UNSUPPORTED_SHAPE;
        Workspace w = carve_dtc(workspace, M, K);
        mmf_status st = launch_quant(x, gamma, eps, M, K, w.q, w.absmax, w.qsum, s, pdl, dev->num_sms, u, NT);
        if (st != MMF_OK) return st;
        return launch_gemv_wide(NT, true, gr, wplan, w, M, K, nullptr, s);
    }
    Workspace w = carve(workspace, M, K);
    mmf_status st = launch_quant(x, gamma, eps, M, K, w.q, w.absmax, w.qsum, s, pdl, dev->num_sms, u);
    if (st != MMF_OK) return st;
    for (int i = 0; i < count; ++i) {
        if (proj[i].N == 0) continue;
        TcParams p{};
        p.qsum = w.qsum;
        p.absmax = w.absmax;
        p.scale = proj[i].scale;
        p.y = proj[i].y;
        p.M = static_cast<int>(M);
        p.K = static_cast<int>(K);
        p.N = static_cast<int>(proj[i].N);
        // only the quantiser may overlap the kernel before it: the contraction
        // reads the codes the quantiser writes, and waits for it either way
        if ((st = launch_tc(true, w.q, proj[i].packed, p, s, pdl, dev->num_sms)) != MMF_OK) return st;
    }
    return MMF_OK;
}

}  // namespace

extern "C" {

const char* mmf_status_string(int status) {
    switch (status) {
        case MMF_OK: return "MMF_OK";
        case MMF_ERR_INVALID_ARG: return "MMF_ERR_INVALID_ARG";
        case MMF_ERR_UNSUPPORTED_SHAPE: return "MMF_ERR_UNSUPPORTED_SHAPE";
        case MMF_ERR_MISALIGNED: return "MMF_ERR_MISALIGNED";
        case MMF_ERR_WORKSPACE: return "MMF_ERR_WORKSPACE";
        case MMF_ERR_CUDA: return "MMF_ERR_CUDA";
        case MMF_ERR_TIMEOUT: return "MMF_ERR_TIMEOUT";
        case MMF_ERR_NO_DEVICE: return "MMF_ERR_NO_DEVICE";
        default: return "MMF_ERR_UNKNOWN";
    }
}

const char* mmf_version(void) { return "mmf 0.1.0 sm_100a"; }

size_t mmf_packed_bytes(int64_t N, int64_t K) {
    if (N < 0 || K < 0) return 0;
    return static_cast<size_t>(N) * static_cast<size_t>(K) / 4;
}

size_t mmf_workspace_bytes(int64_t M, int64_t K, int64_t N) {
    if (check_shape(M, K, N) != MMF_OK || M == 0 || N == 0) return 0;
    if (takes_gemv(M, K)) return 0;
    if (takes_decode_tc(M, K)) return workspace_size_dtc(M, K);
    return workspace_size_tc(M, K);
}

int mmf_fwd_launches(int64_t M, int64_t K, int64_t N, int count) {
    if (check_shape(M, K, N) != MMF_OK || M == 0 || N == 0 || count < 1 || count > MMF_MAX_GROUP) return 0;
    if (takes_gemv(M, K)) return 1;
    if (takes_decode_tc(M, K)) return 2;
    return 1 + count;
}

int mmf_pack_ternary(const float* W, int64_t N, int64_t K, float eps_w, uint32_t* packed, float* scale,
                     void* stream) {
    if (!(eps_w >= 0.0f) || eps_w > 1e30f) return MMF_ERR_INVALID_ARG;
    mmf_status st = check_shape(0, K, N);
    if (st != MMF_OK) return st;
    if (N == 0) return MMF_OK;  // empty: pointers may be NULL, nothing is written
    if (!W || !packed || !scale) return MMF_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(packed) || !aligned16(scale)) return MMF_ERR_MISALIGNED;
    DeviceState* dev;
    if ((st = device_state(&dev)) != MMF_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t n = N * K;
    const int np = absmean_num_partials(n);
    int64_t chunk = (n + np - 1) / np;
    chunk = (chunk + 3) & ~int64_t(3);
    double* partials = reinterpret_cast<double*>(packed);  // scratch: the codes overwrite it below
    absmean_partials_kernel<<<np, kPackThreads, 0, s>>>(W, n, chunk, partials);
    if ((st = launch_status()) != MMF_OK) return st;
    absmean_finalize_kernel<<<1, kPackThreads, 0, s>>>(partials, np, n, scale);
    if ((st = launch_status()) != MMF_OK) return st;
    const int64_t nwords = n / 16;
    int64_t grid = (nwords + kPackThreads - 1) / kPackThreads;
    if (grid > int64_t(dev->num_sms) * 16) grid = int64_t(dev->num_sms) * 16;
    ternary_encode_kernel<<<static_cast<unsigned>(grid), kPackThreads, 0, s>>>(W, nwords, eps_w, scale, packed);
    return launch_status();
}

int mmf_quantize_act(const uint16_t* x, const float* gamma, float eps, int64_t M, int64_t K, int8_t* q,
                     float* absmax, void* stream) {
    if (!(eps >= 0.0f) || eps > 1e30f) return MMF_ERR_INVALID_ARG;
    mmf_status st = check_shape(M, K, 1);
    if (st != MMF_OK) return st;
    if (M == 0) return MMF_OK;
    if (!x || !gamma || !q || !absmax) return MMF_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gamma) || !aligned16(q) || !aligned16(absmax)) return MMF_ERR_MISALIGNED;
    DeviceState* dev;
    if ((st = device_state(&dev)) != MMF_OK) return st;
    return launch_quant(x, gamma, eps, M, K, q, absmax, nullptr, static_cast<cudaStream_t>(stream), false, dev->num_sms);
}

int mmf_ternary_acc(const int8_t* q, const uint32_t* packed, int64_t M, int64_t K, int64_t N, int32_t* acc,
                    void* workspace, size_t workspace_bytes, void* stream) {
    mmf_status st = check_shape(M, K, N);
    if (st != MMF_OK) return st;
    if (M == 0 || N == 0) return MMF_OK;
    if (!q || !packed || !acc) return MMF_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(packed) || !aligned16(acc)) return MMF_ERR_MISALIGNED;
    const size_t need = mmf_workspace_bytes(M, K, N);
    if (need > 0 && (!workspace || workspace_bytes < need)) return MMF_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return MMF_ERR_MISALIGNED;
    DeviceState* dev;
    if ((st = device_state(&dev)) != MMF_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    GemvPlan plan;
    if (M < kDecodeTcMinM && gemv_plan(static_cast<int>(M), static_cast<int>(K), N, dev->num_sms, &plan)) {
        GemvParams p{};
        p.q_in = q;
        p.packed[0] = packed;
        p.acc = acc;
        p.row_start[0] = 0;
        p.row_start[1] = static_cast<int>(N);
        p.nproj = 1;
        p.M = static_cast<int>(M);
        p.K = static_cast<int>(K);
        p.rows_per_stage = plan.rows_per_stage;
        p.rows_per_cta = plan.rows_per_cta;
        p.stage_bytes = plan.stage_bytes;
        p.stages = plan.stages;
        return launch_gemv<false>(p, plan, s, false);
    }
    if (takes_decode_tc(M, K)) {
        const int NT = decode_tc_nt(M);
        WideGroup gr;
        gr.n = 1;
        gr.packed[0] = packed;
        gr.scale[0] = nullptr;
        gr.y[0] = nullptr;
        gr.N[0] = N;
        GemvWidePlan wplan;
        if (!gemv_wide_plan(static_cast<int>(K), NT, gr.slabs(), dev->wide_clusters, &wplan)) return MMF_ERR_UNSUPPORTED_SHAPE;
        Workspace w = carve_dtc(workspace, M, K);
        st = launch(qsum_kernel, dim3(static_cast<unsigned>(NT)), dim3(kQuantThreads), 0, s, false, q,
                    static_cast<int>(K), M, w.qsum, w.q, NT);
        if (st != MMF_OK) return st;
        return launch_gemv_wide(NT, false, gr, wplan, w, M, K, acc, s);
    }
    Workspace w = carve(workspace, M, K);
    st = launch(qsum_kernel, dim3(static_cast<unsigned>(M)), dim3(kQuantThreads), 0, s, false, q, static_cast<int>(K),
                M, w.qsum, static_cast<int8_t*>(nullptr), 0);
    if (st != MMF_OK) return st;
    TcParams p{};
    p.qsum = w.qsum;
    p.acc = acc;
    p.M = static_cast<int>(M);
    p.K = static_cast<int>(K);
    p.N = static_cast<int>(N);
    return launch_tc(false, q, packed, p, s, false, dev->num_sms);
}

int mmf_bitlinear_fwd(const uint16_t* x, const float* gamma, float eps, const uint32_t* packed, const float* scale,
                      int64_t M, int64_t K, int64_t N, uint16_t* y, void* workspace, size_t workspace_bytes,
                      void* stream) {
    if (!(eps >= 0.0f) || eps > 1e30f) return MMF_ERR_INVALID_ARG;
    mmf_status st = check_shape(M, K, N);
    if (st != MMF_OK) return st;
    if (M == 0 || N == 0) return MMF_OK;
    if (!x || !gamma || !packed || !scale || !y) return MMF_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gamma) || !aligned16(packed) || !aligned16(scale) || !aligned16(y))
        return MMF_ERR_MISALIGNED;
    const size_t need = mmf_workspace_bytes(M, K, N);
    if (need > 0 && (!workspace || workspace_bytes < need)) return MMF_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return MMF_ERR_MISALIGNED;
    DeviceState* dev;
    if ((st = device_state(&dev)) != MMF_OK) return st;
    mmf_projection pr;
    pr.packed = packed;
    pr.scale = scale;
    pr.y = y;
    pr.N = N;
    return fwd_impl(x, gamma, eps, M, K, &pr, 1, workspace, 0u, static_cast<cudaStream_t>(stream), dev);
}

// Rows summed per dgamma partial: the fused RMSNorm backward's CTA rows when
// K allows it, else the two-stage column sum's chunk.
int64_t bwd_partial_rows(int64_t K) { return K <= kBwdFusedMaxK ? kBwdFusedRows : kDgammaRows; }

size_t mmf_bwd_workspace_bytes(int64_t M, int64_t K, int64_t N) {
    if (check_shape(M, K, N) != MMF_OK) return 0;
    const size_t m = static_cast<size_t>(M), k = static_cast<size_t>(K);
    const size_t chunks = (m + bwd_partial_rows(K) - 1) / bwd_partial_rows(K);
    // q, absmax, qsum, inv, dr (fp32), dgamma partials (fp64)
    return align256(m * k) + 3 * align256(4 * m) + align256(4 * m * k) + align256(8 * chunks * k);
}

int mmf_bitlinear_bwd(const uint16_t* dy, const uint16_t* x, const float* gamma, float eps, const uint32_t* packed,
                      const float* scale, int64_t M, int64_t K, int64_t N, uint16_t* dx, float* dgamma, float* dW,
                      void* workspace, size_t workspace_bytes, void* stream) {
    if (!(eps >= 0.0f) || eps > 1e30f) return MMF_ERR_INVALID_ARG;
    mmf_status st = check_shape(M, K, N);
    if (st != MMF_OK) return st;
    // dy rows are read by TMA (row pitch a multiple of 16 bytes); beyond the fused
    // RMSNorm backward's K the dgamma row chunks go on grid.y
    if ((N % 8) != 0 || (K > kBwdFusedMaxK && M > 65535L * kDgammaRows)) return MMF_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 && N == 0) return MMF_OK;
    // buffers of an empty extent may be NULL
    if (!gamma || !scale || !dgamma) return MMF_ERR_INVALID_ARG;
    if (M > 0 && (!x || !dx || !workspace)) return MMF_ERR_INVALID_ARG;
    if (N > 0 && !dW) return MMF_ERR_INVALID_ARG;
    if (M > 0 && N > 0 && (!dy || !packed)) return MMF_ERR_INVALID_ARG;
    if (!aligned16(dy) || !aligned16(x) || !aligned16(gamma) || !aligned16(packed) || !aligned16(scale) ||
        !aligned16(dx) || !aligned16(dgamma) || !aligned16(dW) || !aligned16(workspace))
        return MMF_ERR_MISALIGNED;
    if (workspace_bytes < mmf_bwd_workspace_bytes(M, K, N)) return MMF_ERR_WORKSPACE;
    DeviceState* dev;
    if ((st = device_state(&dev)) != MMF_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // workspace: q, absmax, qsum, inv, dr (fp32 [M][K]), dgamma partials
    uint8_t* b = static_cast<uint8_t*>(workspace);
    const size_t m = static_cast<size_t>(M), k = static_cast<size_t>(K);
    int8_t* q = reinterpret_cast<int8_t*>(b);
    b += align256(m * k);
    float* absmax = reinterpret_cast<float*>(b);
    b += align256(4 * m);
    int* qsum = reinterpret_cast<int*>(b);
    b += align256(4 * m);
    float* inv = reinterpret_cast<float*>(b);
    b += align256(4 * m);
    float* dr = reinterpret_cast<float*>(b);
    b += align256(4 * m * k);
    double* part = reinterpret_cast<double*>(b);
    const int chunks = static_cast<int>((M + bwd_partial_rows(K) - 1) / bwd_partial_rows(K));
    const int row_tiles = static_cast<int>(K / kBwRows);

    if (M > 0 && (st = launch_quant(x, gamma, eps, M, K, q, absmax, qsum, s, false, dev->num_sms)) != MMF_OK) return st;
    // dr[M][K] = dy . w~ (an empty contraction when N == 0 gives zeros)
    if (M > 0 && N == 0) {
        if (cudaMemsetAsync(dr, 0, 4 * m * k, s) != cudaSuccess) return MMF_ERR_CUDA;
    } else if (M > 0) {
        CUtensorMap mb, mr;
        if ((st = encode_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dy, N, M, 2 * N, kBwKs, kBwCols,
                            CU_TENSOR_MAP_SWIZZLE_128B)) != MMF_OK)
            return st;
        if ((st = encode_2d(&mr, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, K / 4, N, K / 4, kBwRows / 4, kBwKs,
                            CU_TENSOR_MAP_SWIZZLE_NONE)) != MMF_OK)
            return st;
        BwParams bp{};
        bp.out = dr;
        bp.K = static_cast<int>(K);
        bp.cols = static_cast<int>(M);
        bp.contr = static_cast<int>(N);
        bp.row_tiles = row_tiles;
        bp.num_tiles = row_tiles * static_cast<int>((M + kBwCols - 1) / kBwCols);
        const dim3 grid(static_cast<unsigned>(bp.num_tiles < dev->num_sms ? bp.num_tiles : dev->num_sms));
        if ((st = launch(gemm_bwd_kernel<0>, grid, dim3(kBwThreads), BwLayout<0>::smem_bytes, s, false, mb, mr, bp)) !=
            MMF_OK)
            return st;
    }
    // dW[N][K] = dy^T . (q * absmax / 127) (zeros when M == 0)
    if (N > 0 && M == 0) {
        if (cudaMemsetAsync(dW, 0, 4 * static_cast<size_t>(N) * k, s) != cudaSuccess) return MMF_ERR_CUDA;
    } else if (N > 0) {
        CUtensorMap mb, mr;
        if ((st = encode_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dy, N, M, 2 * N, 64, kBwKs,
                            CU_TENSOR_MAP_SWIZZLE_128B)) != MMF_OK)
            return st;
        if ((st = encode_2d(&mr, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K, M, K, kBwRows, kBwKs,
                            CU_TENSOR_MAP_SWIZZLE_NONE)) != MMF_OK)
            return st;
        BwParams bp{};
        bp.out = dW;
        bp.absmax = absmax;
        bp.K = static_cast<int>(K);
        bp.cols = static_cast<int>(N);
        bp.contr = static_cast<int>(M);
        bp.row_tiles = row_tiles;
        bp.num_tiles = row_tiles * static_cast<int>((N + kBwCols - 1) / kBwCols);
        const dim3 grid(static_cast<unsigned>(bp.num_tiles < dev->num_sms ? bp.num_tiles : dev->num_sms));
        if ((st = launch(gemm_bwd_kernel<1>, grid, dim3(kBwThreads), BwLayout<1>::smem_bytes, s, false, mb, mr, bp)) !=
            MMF_OK)
            return st;
    }
    const auto blocks = [](int64_t count) { return dim3(static_cast<unsigned>((count + kBwdThreads - 1) / kBwdThreads)); };
    if (M > 0 && K <= kBwdFusedMaxK) {
        // dx and the dgamma partials in one pass over x and dr
        const int cpt = static_cast<int>((K / 8 + kBwdThreads - 1) / kBwdThreads);  // 1, 2, 3 or 4
        void (*kern)(const uint16_t*, const float*, const float*, const float*, float, int, int64_t, uint16_t*,
                     double*) = cpt == 1   ? rmsnorm_bwd_fused_kernel<1, 2>
                                : cpt == 2 ? rmsnorm_bwd_fused_kernel<2, 2>
                                : cpt == 3 ? rmsnorm_bwd_fused_kernel<3, 1>
                                           : rmsnorm_bwd_fused_kernel<4, 1>;
        if ((st = launch(kern, dim3(static_cast<unsigned>(chunks)), dim3(kBwdThreads), 0, s, false, x, gamma,
                         static_cast<const float*>(dr), scale, eps, static_cast<int>(K), M, dx, part)) != MMF_OK)
            return st;
    } else if (M > 0) {
        if ((st = launch(rmsnorm_bwd_kernel, dim3(static_cast<unsigned>(M)), dim3(kBwdThreads), 0, s, false, x, gamma,
                         static_cast<const float*>(dr), scale, eps, static_cast<int>(K), dx, inv)) != MMF_OK)
            return st;
        if ((st = launch(dgamma_partial_kernel, dim3(blocks(K).x, static_cast<unsigned>(chunks)), dim3(kBwdThreads), 0,
                         s, false, x, static_cast<const float*>(dr), static_cast<const float*>(inv), M,
                         static_cast<int>(K), part)) != MMF_OK)
            return st;
    }
    return launch(dgamma_final_kernel, dim3(static_cast<unsigned>((K + kDgCols - 1) / kDgCols)), dim3(kDgThreads), 0, s,
                  false, static_cast<const double*>(part), chunks,
                  static_cast<int>(K), scale, dgamma);
}

int mmf_mlgru_scan(const uint16_t* f_pre, const uint16_t* c_pre, const uint16_t* g_pre, const float* h0, int64_t B,
                   int64_t T, int64_t D, uint16_t* o, float* h_last, void* stream) {
    if (B < 0 || T < 0 || D < 0) return MMF_ERR_INVALID_ARG;
    if ((D % 2) != 0 || D > kMaxDim || T > kMaxDim || B > 65535 || B * T * D > (int64_t(1) << 40))
        return MMF_ERR_UNSUPPORTED_SHAPE;
    if (B == 0 || D == 0) return MMF_OK;
    if (T > 0 && (!f_pre || !c_pre || !g_pre || !o)) return MMF_ERR_INVALID_ARG;
    if (T == 0 && !h_last) return MMF_OK;
    if (!aligned16(f_pre) || !aligned16(c_pre) || !aligned16(g_pre) || !aligned16(o) || !aligned16(h0) ||
        !aligned16(h_last))
        return MMF_ERR_MISALIGNED;
    DeviceState* dev;
    mmf_status st = device_state(&dev);
    if (st != MMF_OK) return st;
    const dim3 grid(static_cast<unsigned>((D + 63) / 64), static_cast<unsigned>(B));
    const int64_t rows = B * T;
    if (T > 0 && D % 8 == 0 && D >= kStCh && rows >= kStRows && rows <= int64_t(INT32_MAX) - kStRows) {
        // tensor maps over the [B * T][D] pre-activations: 64 channels x 128 tokens per copy
        CUtensorMap mf, mc, mg;
        if ((st = encode_2d(&mf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f_pre, D, rows, 2 * D, kStCh, kStRows,
                            CU_TENSOR_MAP_SWIZZLE_NONE)) != MMF_OK ||
            (st = encode_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c_pre, D, rows, 2 * D, kStCh, kStRows,
                            CU_TENSOR_MAP_SWIZZLE_NONE)) != MMF_OK ||
            (st = encode_2d(&mg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g_pre, D, rows, 2 * D, kStCh, kStRows,
                            CU_TENSOR_MAP_SWIZZLE_NONE)) != MMF_OK)
            return st;
        return launch(mlgru_scan_tma_kernel, grid, dim3(kStThreads), kStSmemBytes, static_cast<cudaStream_t>(stream),
                      false, mf, mc, mg, h0, static_cast<int>(T), static_cast<int>(D), o, h_last);
    }
    return launch(mlgru_scan_kernel, grid, dim3(kScanWarps * 32), 0, static_cast<cudaStream_t>(stream), false, f_pre,
                  c_pre, g_pre, h0, static_cast<int>(T), static_cast<int>(D), o, h_last);
}

int mmf_bitlinear_fwd_glu(const uint16_t* g, const uint16_t* u, const float* gamma, float eps,
                          const uint32_t* packed, const float* scale, int64_t M, int64_t K, int64_t N, uint16_t* y,
                          void* workspace, size_t workspace_bytes, unsigned flags, void* stream) {
    if (!(eps >= 0.0f) || eps > 1e30f) return MMF_ERR_INVALID_ARG;
    if (flags & ~MMF_FWD_PDL) return MMF_ERR_INVALID_ARG;
    mmf_status st = check_shape(M, K, N);
    if (st != MMF_OK) return st;
    if (M == 0 || N == 0) return MMF_OK;
    if (!g || !u || !gamma || !packed || !scale || !y) return MMF_ERR_INVALID_ARG;
    if (!aligned16(g) || !aligned16(u) || !aligned16(gamma) || !aligned16(packed) || !aligned16(scale) ||
        !aligned16(y))
        return MMF_ERR_MISALIGNED;
    const size_t need = mmf_workspace_bytes(M, K, N);
    if (need > 0 && (!workspace || workspace_bytes < need)) return MMF_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return MMF_ERR_MISALIGNED;
    DeviceState* dev;
    if ((st = device_state(&dev)) != MMF_OK) return st;
    mmf_projection pr;
    pr.packed = packed;
    pr.scale = scale;
    pr.y = y;
    pr.N = N;
    return fwd_impl(g, gamma, eps, M, K, &pr, 1, workspace, flags, static_cast<cudaStream_t>(stream), dev, u);
}

int mmf_bitlinear_fwd_group(const uint16_t* x, const float* gamma, float eps, int64_t M, int64_t K,
                            const mmf_projection* proj, int count, void* workspace, size_t workspace_bytes,
                            unsigned flags, void* stream) {
    if (!(eps >= 0.0f) || eps > 1e30f) return MMF_ERR_INVALID_ARG;
    if (!proj || count < 1 || count > MMF_MAX_GROUP) return MMF_ERR_INVALID_ARG;
    if ((flags & ~static_cast<unsigned>(MMF_FWD_PDL)) != 0) return MMF_ERR_INVALID_ARG;
    int64_t R = 0;
    for (int i = 0; i < count; ++i) {
        if (proj[i].N < 0) return MMF_ERR_INVALID_ARG;
        R += proj[i].N;
    }
    mmf_status st = check_shape(M, K, R);
    if (st != MMF_OK) return st;
    if (M == 0 || R == 0) return MMF_OK;
    if (!x || !gamma) return MMF_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gamma)) return MMF_ERR_MISALIGNED;
    for (int i = 0; i < count; ++i) {
        if (proj[i].N == 0) continue;
        if (!proj[i].packed || !proj[i].scale || !proj[i].y) return MMF_ERR_INVALID_ARG;
        if (!aligned16(proj[i].packed) || !aligned16(proj[i].scale) || !aligned16(proj[i].y))
            return MMF_ERR_MISALIGNED;
    }
    const size_t need = mmf_workspace_bytes(M, K, R);
    if (need > 0 && (!workspace || workspace_bytes < need)) return MMF_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return MMF_ERR_MISALIGNED;
    DeviceState* dev;
    if ((st = device_state(&dev)) != MMF_OK) return st;
    return fwd_impl(x, gamma, eps, M, K, proj, count, workspace, flags, static_cast<cudaStream_t>(stream), dev);
}

int mmf_bitlinear_fwd_noalloc(const uint16_t* x, const float* gamma, float eps, const uint32_t* packed,
                              const float* scale, int64_t M, int64_t K, int64_t N, uint16_t* y, void* stream) {
    if (!(eps >= 0.0f) || eps > 1e30f) return MMF_ERR_INVALID_ARG;
    mmf_status st = check_shape(M, K, N);
    if (st != MMF_OK) return st;
    if (M == 0 || N == 0) return MMF_OK;
    if (!x || !gamma || !packed || !scale || !y) return MMF_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gamma) || !aligned16(packed) || !aligned16(scale) || !aligned16(y))
        return MMF_ERR_MISALIGNED;
    const size_t need = mmf_workspace_bytes(M, K, N);
    if (need > kNoAllocScratchBytes) return MMF_ERR_WORKSPACE;  // larger than the static scratch
    DeviceState* dev;
    if ((st = device_state(&dev)) != MMF_OK) return st;
    void* ws = nullptr;
    if (need > 0) {
        int d = 0;
        if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return MMF_ERR_NO_DEVICE;
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_noalloc_scratch_ptr[d]) {
            // once per device, with that device current
            void* ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return MMF_ERR_CUDA;
            g_noalloc_scratch_ptr[d] = ptr;
        }
        ws = g_noalloc_scratch_ptr[d];
    }
    // Nothing in the scratch has to start at zero: the quantiser writes every
    // code, absmax and sum the contraction reads, on each call.
    mmf_projection pr;
    pr.packed = packed;
    pr.scale = scale;
    pr.y = y;
    pr.N = N;
    return fwd_impl(x, gamma, eps, M, K, &pr, 1, ws, 0u, static_cast<cudaStream_t>(stream), dev);
}

int mmf_hbm_copy(const void* src, void* dst, size_t bytes, void* stream) {
    if (!src || !dst) return MMF_ERR_INVALID_ARG;
    if ((bytes & 15u) != 0) return MMF_ERR_INVALID_ARG;
    if (!aligned16(src) || !aligned16(dst)) return MMF_ERR_MISALIGNED;
    if (bytes == 0) return MMF_OK;
    DeviceState* dev;
    mmf_status st = device_state(&dev);
    if (st != MMF_OK) return st;
    const int64_t n16 = static_cast<int64_t>(bytes / 16);
    int64_t grid = (n16 + kCopyThreads - 1) / kCopyThreads;
    if (grid > int64_t(dev->num_sms) * 4) grid = int64_t(dev->num_sms) * 4;
    hbm_copy_kernel<<<static_cast<unsigned>(grid), kCopyThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), n16);
    return launch_status();
}

int mmf_selftest_timeout(uint64_t limit_ns, int32_t* waited_out, void* stream) {
    if (limit_ns == 0 || limit_ns > kWaitLimitNs) return MMF_ERR_INVALID_ARG;
    if (waited_out && (reinterpret_cast<uintptr_t>(waited_out) & 3u)) return MMF_ERR_MISALIGNED;
    DeviceState* dev;
    mmf_status st = device_state(&dev);
    if (st != MMF_OK) return st;
    selftest_timeout_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, waited_out);
    return launch_status();
}

int mmf_check_async(void* stream) {
    DeviceState* dev;
    mmf_status st = device_state(&dev);
    if (st != MMF_OK) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MMF_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, mmf::g_error_word, sizeof(word)) != cudaSuccess) return MMF_ERR_CUDA;
    if (word != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(mmf::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return MMF_ERR_CUDA;
        return MMF_ERR_TIMEOUT;
    }
    return MMF_OK;
}

}  // extern "C"
