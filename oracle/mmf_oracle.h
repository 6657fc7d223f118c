/*
 * mmf_oracle.h -- plain CPU oracle for the fused RMSNorm + BitLinear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path (the
 * CUDA library and its Python binding) never calls into it, and the two share
 * no source, header, table or helper.
 *
 * What it computes is the definition of the BitLinear layer of the MatMul-free
 * language model ("Scalable MatMul-free Language Modeling", Zhu et al., as
 * described by the jiqizhixin.com article, section "具有三值权重的 MatMul-free
 * 密集层" with its Algorithm 1 (fused RMSNorm + BitLinear), and by the
 * datacamp.com article, section "Thay MatMul bằng các phép toán tam phân" and
 * the "RMS norm" item of its component figure).  The pages print no formula,
 * so every step below is the plain reading written out in each function's
 * comment.
 *
 * Layouts (all row-major, no padding):
 *   W      fp32  [N][K]   latent weights, y = x . W~^T (nn.Linear convention)
 *   wt     int8  [N][K]   ternary weights in {-1, 0, +1}
 *   packed uint32[N][K/16] 2-bit codes; see orc_encode_packed
 *   x      bf16  [M][K]   activations, passed as raw uint16 bit patterns
 *   gamma  fp32  [K]      RMSNorm gain
 *   q      int8  [M][K]   activation codes in [-127, 127]
 *   absmax fp32  [M]      per-token max |r| (dequantisation factor absmax/127)
 *   acc    int32 [M][N]
 *   y      bf16  [M][N]   raw uint16 bit patterns
 *
 * Error behaviour: none of these functions checks its arguments; the caller
 * passes valid buffers of the sizes above.  The functions are sequential except
 * orc_ternary_acc, whose (token, output row) pairs may be shared out among
 * OpenMP threads (the result does not depend on the thread count: every acc
 * element is a plain integer sum formed by one thread).
 */
#ifndef MMF_ORACLE_H
#define MMF_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* bf16 bit pattern -> fp32 (exact). */
float orc_bf16_to_f32(uint16_t b);
/* fp64 -> bf16 with round-to-nearest, ties to even, computed from the
 * definition (8 significant bits, fp32 exponent range, subnormals kept). */
uint16_t orc_f64_to_bf16(double v);

/* Absmean ternarisation (A1): beta = mean|W| summed in fp64 and rounded to
 * fp32; wt = clamp(rint(W / (beta + eps_w)), -1, 1) with the division taken in
 * fp32 (the precision in which the code is decided). */
void orc_absmean_ternary(const float* W, int64_t N, int64_t K, float eps_w,
                         int8_t* wt, float* beta);

/* 2-bit packing of ternary weights (the library's storage format).
 * K must be a multiple of 16.  Word j of row n holds weights k = 16j + i for
 * i = 0..15; weight i sits in bits [8*(i%4) + 2*(i/4), +2) and its code is
 * wt + 1 (0 -> -1, 1 -> 0, 2 -> +1; 3 is never written). */
void orc_encode_packed(const int8_t* wt, int64_t N, int64_t K, uint32_t* packed);
/* Inverse of orc_encode_packed.  Returns the number of codes equal to 3 found
 * (which no valid packed matrix contains); those entries decode to 0. */
int64_t orc_decode_packed(const uint32_t* packed, int64_t N, int64_t K, int8_t* wt);

/* RMSNorm followed by per-token absmax int8 quantisation (A3, A4):
 *   ms = (float)(sum_k x_k^2 / K)           sum and quotient in fp64
 *   inv = 1 / sqrt(ms + eps)                 fp32, correctly rounded
 *   r_k = (x_k * inv) * gamma_k              fp32, two roundings, this order
 *   absmax = max(max_k |r_k|, 1e-5)
 *   s = 127 / absmax                         fp32, correctly rounded
 *   q_k = clamp(rint(r_k * s), -127, 127)    fp32 product, ties to even
 * The fp32 part is where a float decides an integer code, so it is taken in
 * the precision the CUDA path uses. */
void orc_rmsnorm_quant(const uint16_t* x, const float* gamma, float eps,
                       int64_t M, int64_t K, int8_t* q, float* absmax);

/* Ternary accumulation (A2): acc[m][n] = sum over k with wt=+1 of q minus the
 * sum over k with wt=-1 of q; a 0 weight contributes nothing.  int32. */
void orc_ternary_acc(const int8_t* q, const int8_t* wt, int64_t M, int64_t K,
                     int64_t N, int32_t* acc);

/* Rescale (A5): y = bf16_rn(acc * (absmax / 127) * beta), evaluated in fp64
 * and rounded once to bf16. */
void orc_rescale(const int32_t* acc, const float* absmax, float beta,
                 int64_t M, int64_t N, uint16_t* y);

/* The whole layer from latent weights: ternarise W, quantise x, accumulate,
 * rescale.  Scratch for wt (N*K bytes), q (M*K bytes), absmax (M floats) and
 * acc (M*N int32) is allocated and freed inside.  Returns 0, or -1 if an
 * allocation failed. */
int orc_bitlinear(const uint16_t* x, const float* gamma, float eps,
                  const float* W, float eps_w, int64_t M, int64_t K, int64_t N,
                  uint16_t* y, float* beta_out);

/* The gated product of the GLU channel mixer, the input of its down
 * projection (datacamp.com, section "Các thành phần lõi: MLGRU và GLU": one
 * BitLinear output goes through SiLU and is multiplied element-wise by the
 * other).  p = bf16_rn(SiLU(g) * u), SiLU(v) = v * (1 / (1 + e^-v)), each
 * step rounded to fp32 (the precision the CUDA path takes this decision in);
 * g, u, p bf16 [n]. */
void orc_glu_gate(const uint16_t* g, const uint16_t* u, int64_t n, uint16_t* p);

/* The MLGRU token mixer's element-wise recurrence (datacamp.com, section
 * "Các thành phần lõi: MLGRU và GLU": tokens are taken one at a time; gates
 * with values between 0 and 1 decide how much of the previous hidden state and
 * of the current token is kept; jiqizhixin.com, section "MatMul-free 语言模型
 * 架构", whose formulas are stripped).  For every sequence b and channel k,
 * from h = h0[b][k] (0 when h0 is NULL), token by token:
 *   f = sigma(f_pre), c = SiLU(c_pre), g = sigma(g_pre),  sigma(v) = 1 / (1 + e^-v),
 *   h = f * h + (1 - f) * c,  o = bf16_rn(g * h)
 * every step rounded to fp32; h_last[b][k] = h after the last token.
 * f_pre, c_pre, g_pre, o: bf16 [B][T][D]; h0, h_last: fp32 [B][D]. */
void orc_mlgru_scan(const uint16_t* f_pre, const uint16_t* c_pre, const uint16_t* g_pre,
                    const float* h0, int64_t B, int64_t T, int64_t D, uint16_t* o, float* h_last);

/* Backward of the fused BitLinear layer with the straight-through estimator
 * (ld246.com, section "训练与优化：新的策略": the non-differentiable ternary
 * weights and quantisation are back-propagated with a surrogate gradient, the
 * straight-through estimator, read as passing gradients through the
 * quantisers unchanged).  Forward: r = RMSNorm(x) *
 * gamma, x_q = q * (absmax / 127) (the quantised r), W_q = w~ * beta,
 * y = x_q . W_q^T.  With both quantisers taken as the identity:
 *   dr[m][k]  = sum_n dy[m][n] * W_q[n][k]
 *   dW[n][k]  = sum_m dy[m][n] * x_q[m][k]
 *   dgamma[k] = sum_m dr[m][k] * x[m][k] * inv_m
 *   dx[m][k]  = inv_m * gamma[k] * dr[m][k]
 *               - x[m][k] * inv_m^3 * (sum_j gamma[j] dr[m][j] x[m][j]) / K
 * with inv_m = 1 / sqrt(sum_k x^2 / K + eps); all in fp64, dx rounded to
 * bf16.  q and absmax are the forward's (orc_rmsnorm_quant).
 * dy bf16 [M][N]; x bf16 [M][K]; wt int8 [N][K]; dx bf16 [M][K];
 * dgamma fp32 [K]; dW fp32 [N][K].  Returns 0, or -1 if scratch allocation
 * failed. */
int orc_bitlinear_bwd(const uint16_t* dy, const uint16_t* x, const float* gamma, float eps,
                      const int8_t* wt, float beta, int64_t M, int64_t K, int64_t N,
                      uint16_t* dx, float* dgamma, float* dW);

/* Number of OpenMP threads orc_ternary_acc uses (1 when built without OpenMP). */
int orc_num_threads(void);

#ifdef __cplusplus
}
#endif

#endif /* MMF_ORACLE_H */
