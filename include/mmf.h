/*
 * mmf.h -- C ABI of the fused RMSNorm + BitLinear library for NVIDIA B200
 * (sm_100a).  Library: bitlinear_rmsnorm_quant_b200/libmmf.so.
 *
 * The layer is the BitLinear dense layer of the MatMul-free language model
 * ("Scalable MatMul-free Language Modeling", Zhu et al.):
 *   - weights are ternary {-1, 0, +1}, obtained from full-precision latent
 *     weights by absmean quantisation (datacamp.com, section "Thay MatMul bằng
 *     các phép toán tam phân"; jiqizhixin.com, section "具有三值权重的
 *     MatMul-free 密集层"), so the product needs only additions and
 *     subtractions (ld246.com, section "三值权重的应用");
 *   - the activations pass through RMSNorm before quantisation (datacamp.com,
 *     component figure, item "RMS norm"), and RMSNorm and quantisation are one
 *     fused operation that reads x from HBM once (ld246.com, section "融合
 *     BitLinear 层的创新"; jiqizhixin.com, Algorithm 1);
 *   - activations are quantised per token to int8 by absmax, accumulated in
 *     int32, and rescaled by (absmax/127) * mean|W|.  The pages give no
 *     formula; these are the plain definitions, stated per function below.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers owned by the caller unless stated.  The
 *     library never allocates, frees or caches device memory and keeps no
 *     pointer after a call returns.
 *   - Every pointer must be 16-byte aligned (TMA and 128-bit loads).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous and ordered on that stream; results
 *     are ready when the stream has reached the call.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Shapes: M tokens (0 <= M <= 16,776,960 = 65535 * 256; the scan states
 *     its own sizes), K = d_in (128 <= K <= 65536,
 *     K % 128 == 0), N = d_out (0 <= N < 2^31).  M == 0 or N == 0 is a no-op
 *     returning MMF_OK once the scalar arguments and K are valid; the buffer
 *     pointers of an empty problem are not checked and may be NULL.
 *   - Argument errors return synchronously and launch nothing.  A failed
 *     launch returns MMF_ERR_CUDA.  A device-side wait that timed out (every
 *     wait inside the kernels is bounded, about one second) is recorded in a
 *     device error word, and the kernel that gave up returns without writing
 *     its outputs; mmf_check_async reports (MMF_ERR_TIMEOUT) and clears it.
 *   - The first call on a device does a one-time set-up (device properties,
 *     kernel attributes, the driver's tensor-map entry point); make that
 *     first call outside any CUDA graph capture.
 *   - Entry points are thread-safe; calls that overlap on the GPU must not
 *     write the same output or workspace buffer.
 */
#ifndef MMF_H
#define MMF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mmf_status {
    MMF_OK = 0,
    MMF_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad eps */
    MMF_ERR_UNSUPPORTED_SHAPE = 2, /* K not a multiple of 128 in [128, 65536], or too large */
    MMF_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned */
    MMF_ERR_WORKSPACE = 4,         /* workspace missing or smaller than mmf_workspace_bytes */
    MMF_ERR_CUDA = 5,              /* a CUDA runtime call or launch failed */
    MMF_ERR_TIMEOUT = 6,           /* a bounded device-side wait ran out */
    MMF_ERR_NO_DEVICE = 7          /* no sm_100 device is current */
} mmf_status;

/* Human-readable name of a status code; never NULL. */
const char* mmf_status_string(int status);

/* Library version string, e.g. "mmf 0.1.0 sm_100a". */
const char* mmf_version(void);

/* Number of kernel launches one mmf_bitlinear_fwd_group call with `count`
 * non-empty projections of N rows in total issues for this (M, K): 1 on the
 * fused decode path (1 .. 3 tokens), 2 (quantiser + contraction) for
 * 4 .. 32 tokens, 1 + count on the large-M path; 0 for an invalid or empty
 * shape.  A single mmf_bitlinear_fwd is count = 1. */
int mmf_fwd_launches(int64_t M, int64_t K, int64_t N, int count);

/* Bytes of the packed ternary matrix for an N x K weight: N * K / 4. */
size_t mmf_packed_bytes(int64_t N, int64_t K);

/* Bytes of device workspace mmf_bitlinear_fwd and mmf_ternary_acc need for
 * this shape; 0 when the shape takes the fused decode path (1 .. 3 tokens),
 * which needs none.  For 4 .. 32 tokens it holds the codes in the decode
 * tensor-core kernel's operand layout (16 or 32 token rows per 128-wide K
 * chunk) and the per-token absmax and code sums; for more tokens the codes in
 * row-major order and the same sums.  Depends only on (M, K, N). */
size_t mmf_workspace_bytes(int64_t M, int64_t K, int64_t N);

/*
 * mmf_pack_ternary -- absmean ternarisation and 2-bit packing of a latent
 * weight matrix (datacamp.com, "Thay MatMul bằng các phép toán tam phân": the
 * full-precision weights are scaled by their mean absolute value and rounded
 * to the nearest of -1, 0, +1; read as a division, since a product would round
 * every weight of a N(0, 0.02) matrix to 0).
 *
 *   beta   = mean over all N*K of |W|, summed in fp64 in a fixed order and
 *            rounded once to fp32; written to scale[0].
 *   w~     = clamp(rint(W / (beta + eps_w)), -1, 1), the division in fp32
 *            (IEEE, round to nearest even), rint ties to even.
 *   packed = uint32 [N][K/16], row-major, row pitch K/4 bytes.  Word j of row n
 *            holds weights k = 16j + i, i = 0..15; weight i occupies bits
 *            [8*(i%4) + 2*(i/4), +2) and stores the code w~ + 1
 *            (0 = -1, 1 = 0, 2 = +1; 3 is never written).
 *
 * W: fp32 [N][K] row-major (nn.Linear layout, y = x W~^T).  eps_w >= 0.
 * `packed` is also used as scratch before it receives the codes, so it must
 * not alias W.  Deterministic: the same W gives the same bits on every run.
 */
int mmf_pack_ternary(const float* W, int64_t N, int64_t K, float eps_w,
                     uint32_t* packed, float* scale, void* stream);

/*
 * mmf_quantize_act -- RMSNorm followed by per-token absmax int8 quantisation,
 * one fused pass over x (the same arithmetic as inside mmf_bitlinear_fwd):
 *   ms     = (float)(sum_k x_k^2 / K)      sum and quotient in fp64
 *   inv    = 1 / sqrt(ms + eps)            fp32, correctly rounded
 *   r_k    = (x_k * inv) * gamma_k         fp32, two roundings in this order
 *   absmax = max(max_k |r_k|, 1e-5)        written to absmax[m]
 *   q_k    = clamp(rint(r_k * (127/absmax)), -127, 127)
 * x: bf16 [M][K]; gamma: fp32 [K]; q: int8 [M][K]; absmax: fp32 [M].
 * eps >= 0.  x and q must not alias.
 */
int mmf_quantize_act(const uint16_t* x, const float* gamma, float eps,
                     int64_t M, int64_t K, int8_t* q, float* absmax, void* stream);

/*
 * mmf_ternary_acc -- the ternary contraction alone, for parity checks:
 *   acc[m][n] = sum over k with w~[n][k] = +1 of q[m][k]
 *             - sum over k with w~[n][k] = -1 of q[m][k]      (int32, exact)
 * q: int8 [M][K] (values in [-127, 127]); packed as from mmf_pack_ternary;
 * acc: int32 [M][N].  Takes the same kernel path mmf_bitlinear_fwd takes for
 * this (M, K, N), so it needs the same workspace.
 */
int mmf_ternary_acc(const int8_t* q, const uint32_t* packed, int64_t M,
                    int64_t K, int64_t N, int32_t* acc, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * mmf_bitlinear_fwd -- the fused BitLinear forward:
 *   (q, absmax) = RMSNorm + quantisation of x, as in mmf_quantize_act
 *   acc         = ternary contraction of q with the packed weights
 *   y[m][n]     = bf16_rn((float)acc[m][n] * ((absmax[m] / 127) * scale[0]))
 * x: bf16 [M][K]; gamma: fp32 [K]; packed/scale as from mmf_pack_ternary;
 * y: bf16 [M][N].  workspace: device buffer of at least
 * mmf_workspace_bytes(M, K, N) bytes (may be NULL when that is 0); it holds
 * the int8 codes between the two kernels of the large-M path.  x, y and the
 * workspace must not overlap.
 */
int mmf_bitlinear_fwd(const uint16_t* x, const float* gamma, float eps,
                      const uint32_t* packed, const float* scale, int64_t M,
                      int64_t K, int64_t N, uint16_t* y, void* workspace,
                      size_t workspace_bytes, void* stream);

/*
 * mmf_bitlinear_fwd_glu -- the down projection of the GLU channel mixer with
 * its gating fused in (datacamp.com, section "Các thành phần lõi: MLGRU và
 * GLU": the input goes through two BitLinear layers, one output through
 * SiLU, multiplied element-wise by the other, and the product through a
 * third BitLinear layer).  The input of the fused forward is
 *   p[m][k] = bf16_rn(SiLU(g[m][k]) * u[m][k]),  SiLU(v) = v * (1 / (1 + e^-v)),
 * each step rounded to fp32; then as mmf_bitlinear_fwd with x = p.  p never
 * goes to memory: the kernels form it while normalising.
 * g, u: bf16 [M][K] (the gate and up projections' outputs); other arguments,
 * workspace (mmf_workspace_bytes(M, K, N)) and errors as mmf_bitlinear_fwd;
 * flags: 0 or MMF_FWD_PDL (g and u are then read only after the kernel before
 * has finished, like x).  g, u, y and the workspace must not overlap.
 */
int mmf_bitlinear_fwd_glu(const uint16_t* g, const uint16_t* u,
                          const float* gamma, float eps, const uint32_t* packed,
                          const float* scale, int64_t M, int64_t K, int64_t N,
                          uint16_t* y, void* workspace, size_t workspace_bytes,
                          unsigned flags, void* stream);

/*
 * mmf_mlgru_scan -- the MLGRU token mixer's element-wise recurrence between
 * its f/c/g projections and its o projection (datacamp.com, section "Các
 * thành phần lõi: MLGRU và GLU": tokens taken one at a time, gates in (0, 1)
 * deciding how much of the previous hidden state and of the current token is
 * kept).  For every sequence b and channel k, from h = h0[b][k] (0 when h0 is
 * NULL), token by token:
 *   f = sigma(f_pre), c = SiLU(c_pre), g = sigma(g_pre),  sigma(v) = 1/(1 + e^-v)
 *   h = f * h + (1 - f) * c          (fp32)
 *   o[b][t][k] = bf16_rn(g * h)      (the o projection's input)
 * and h_last[b][k] = h after the last token (may be NULL).  Tokens are split
 * into chunks combined through their linear maps h -> A h + B, and sigma uses
 * the hardware exponential and reciprocal (a few ulp), so the result matches
 * the token-by-token recurrence to a few fp32 ulps per token, not bit for bit.
 * f_pre, c_pre, g_pre, o: bf16 [B][T][D] (the projections' y layout with
 * M = B * T); h0, h_last: fp32 [B][D].  D must be even, B <= 65535; pointers
 * 16-byte aligned; o must not overlap the inputs.  T = 0 copies h0 (or zeros)
 * to h_last.
 */
int mmf_mlgru_scan(const uint16_t* f_pre, const uint16_t* c_pre,
                   const uint16_t* g_pre, const float* h0, int64_t B, int64_t T,
                   int64_t D, uint16_t* o, float* h_last, void* stream);

/*
 * mmf_bitlinear_bwd -- backward of mmf_bitlinear_fwd with the straight-through
 * estimator (ld246.com, section "训练与优化：新的策略": the non-differentiable
 * ternary weights and quantisation are back-propagated with a surrogate
 * gradient, read as passing gradients through both quantisers unchanged).
 * With x_q = q * (absmax / 127) (the forward's codes) and W_q = w~ * beta:
 *   dr = dy . W_q,  dW = dy^T . x_q,
 *   dx = inv * gamma * dr - x * inv^3 * (sum_k gamma_k dr_k x_k) / K,
 *   dgamma = sum over tokens of dr * x * inv,  inv = 1 / sqrt(sum x^2 / K + eps).
 * dy: bf16 [M][N]; x, gamma, eps, packed, scale as for the forward;
 * dx: bf16 [M][K]; dgamma: fp32 [K]; dW: fp32 [N][K] (the latent weights'
 * gradient); all overwritten.  The two products run on the tensor cores in
 * this library's own kernel (bf16 operands, fp32 accumulation): for dr the
 * ternary weights are unpacked from the 2-bit codes (exact), for dW each
 * token's codes are scaled by absmax / 127 and rounded to bf16 as they are
 * loaded.  An empty contraction gives zeros (M == 0: dW = 0, dgamma = 0;
 * N == 0: dx = 0).  workspace: at least mmf_bwd_workspace_bytes(M, K, N)
 * bytes, no initialisation needed.  Sizes as the forward, with N a multiple
 * of 8 (dy rows are read by TMA), and M <= 4194240 when K > 8192; buffers of an empty extent
 * (x, dx and workspace when M == 0; dW when N == 0; dy and packed when either
 * is 0) may be NULL.
 */
size_t mmf_bwd_workspace_bytes(int64_t M, int64_t K, int64_t N);
int mmf_bitlinear_bwd(const uint16_t* dy, const uint16_t* x, const float* gamma,
                      float eps, const uint32_t* packed, const float* scale,
                      int64_t M, int64_t K, int64_t N, uint16_t* dx,
                      float* dgamma, float* dW, void* workspace,
                      size_t workspace_bytes, void* stream);

/* Flags of mmf_bitlinear_fwd_group. */
#define MMF_FWD_PDL 1u   /* launch as a programmatic dependent of the kernel before it on the stream (see below) */
#define MMF_MAX_GROUP 8  /* projections per mmf_bitlinear_fwd_group call */

/* One projection of a group: its packed weights and scale (as from
 * mmf_pack_ternary for an N x K matrix) and its output y, bf16 [M][N]. */
typedef struct mmf_projection {
    const uint32_t* packed;
    const float* scale;
    uint16_t* y;
    int64_t N;
} mmf_projection;

/*
 * mmf_bitlinear_fwd_group -- the fused forward of `count` (1..MMF_MAX_GROUP)
 * projections that read the same x: the token mixer's gate projections and
 * the channel mixer's gate/up pair each share one normalised, quantised input
 * (jiqizhixin.com, section "MatMul-free 语言模型架构"; datacamp.com, section
 * "Các thành phần lõi: MLGRU và GLU").  x is normalised and quantised once;
 * each projection i then gets y_i exactly as mmf_bitlinear_fwd would compute
 * it (same bits).  On the small-M path all projections run in one launch.
 *
 * proj: HOST array of `count` descriptors (read during the call only); an
 * entry with N == 0 is skipped.  workspace: at least
 * mmf_workspace_bytes(M, K, sum of N) bytes.
 *
 * flags: 0 or MMF_FWD_PDL.  With MMF_FWD_PDL the kernels are launched as
 * programmatic dependents of the kernel before them on the stream: packed
 * weights, scales and gamma are fetched BEFORE that kernel has finished (x is
 * read, and y written, only after it), so the caller guarantees that the
 * immediately preceding kernel on the stream does not write packed, scale or
 * gamma.  Without the flag the launches are ordinary stream-ordered launches.
 */
int mmf_bitlinear_fwd_group(const uint16_t* x, const float* gamma, float eps,
                            int64_t M, int64_t K, const mmf_projection* proj,
                            int count, void* workspace, size_t workspace_bytes,
                            unsigned flags, void* stream);

/*
 * mmf_bitlinear_fwd_noalloc -- mmf_bitlinear_fwd without a caller-supplied
 * workspace; nothing on the pages corresponds to it (it is an interface
 * convenience, not part of the method).
 *
 * Some callers cannot allocate device memory: a plug-in hosted by another
 * runtime that owns all device memory through its own pool (a raw cudaMalloc
 * would bypass that pool's accounting and may fail or fragment it), or a
 * latency-critical caller that must not block in cudaMalloc / cudaFree, which
 * can synchronise the device.  This entry point serves them: the caller passes
 * only inputs and outputs, exactly as for mmf_bitlinear_fwd (same arguments
 * minus the workspace, same results bit for bit), and the large-M workspace
 * comes from a static device array inside the library instead.
 *
 * Limits and behaviour:
 *   - The static scratch holds MMF_NOALLOC_SCRATCH_BYTES bytes (64 MiB);
 *     shapes with mmf_workspace_bytes(M, K, N) above that return
 *     MMF_ERR_WORKSPACE and launch nothing.  Every GPU that loads the library
 *     holds the 64 MiB until the process exits.
 *   - No call allocates or frees device memory.
 *   - The first call on a device (with a workspace-needing shape) looks up
 *     the scratch's device address for that device; make that first call
 *     before any stream capture on the device.
 *   - All calls on a device share the one scratch array.  Calls whose kernels
 *     overlap on the GPU (different streams, or threads with their own
 *     streams) race on it and give wrong results; order them, e.g. on one
 *     stream.  Nothing in the scratch needs clearing between calls: each call
 *     rewrites every byte it reads.
 */
#define MMF_NOALLOC_SCRATCH_BYTES (64u << 20)
int mmf_bitlinear_fwd_noalloc(const uint16_t* x, const float* gamma, float eps,
                              const uint32_t* packed, const float* scale,
                              int64_t M, int64_t K, int64_t N, uint16_t* y,
                              void* stream);

/*
 * mmf_hbm_copy -- streaming device-to-device copy of `bytes` bytes (a multiple
 * of 16) with 128-bit loads and stores.  Measurement kernel: it gives the HBM
 * bandwidth the roofline fractions are stated against.  src and dst must not
 * overlap.
 */
int mmf_hbm_copy(const void* src, void* dst, size_t bytes, void* stream);

/*
 * mmf_selftest_timeout -- failure-detection self-test (no counterpart on the
 * pages).  Launches one thread that waits on a shared-memory barrier nothing
 * arrives at, with the same bounded wait the kernels use but a limit of
 * limit_ns (0 < limit_ns <= 1e9).  The wait gives up, records a timeout in the
 * device error word (so the next mmf_check_async returns MMF_ERR_TIMEOUT),
 * writes 1 to *waited_out if waited_out is not NULL (device pointer, 4-byte
 * aligned), and the kernel returns.  Nothing hangs or faults.
 */
int mmf_selftest_timeout(uint64_t limit_ns, int32_t* waited_out, void* stream);

/*
 * mmf_check_async -- synchronises `stream`, then reads and clears the device
 * error word of the current device.  Returns MMF_ERR_TIMEOUT if a bounded
 * wait in any earlier kernel ran out, MMF_ERR_CUDA if the stream reports an
 * error, else MMF_OK.
 */
int mmf_check_async(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MMF_H */
