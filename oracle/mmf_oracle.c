/*
 * mmf_oracle.c -- plain, slow CPU oracle for the fused RMSNorm + BitLinear
 * layer.  TEST INFRASTRUCTURE ONLY: loaded by the test suite, the smoke check
 * and the benchmark's CPU baseline leg, never by the product path.
 *
 * Every function is the plain definition of one step, written in the order the
 * pages give the steps:
 *   - absmean ternary weights (datacamp.com, "Thay MatMul bằng các phép toán
 *     tam phân": latent full-precision weights are scaled by their mean
 *     absolute value and rounded to the nearest of -1, 0, +1; the page says
 *     "multiplies", read as divides, see orc_absmean_ternary);
 *   - ternary accumulation (ld246.com, "三值权重的应用": +1 adds the input,
 *     -1 subtracts it, 0 does nothing; jiqizhixin.com, "具有三值权重的
 *     MatMul-free 密集层");
 *   - RMSNorm ahead of activation quantisation (datacamp.com, component
 *     figure, item "RMS norm"; jiqizhixin.com, Algorithm 1, fused RMSNorm +
 *     BitLinear, whose flowchart is missing from the page);
 *   - per-token absmax int8 activations and the rescale by absmax/127 times
 *     mean|W| (not printed on the pages; the plain reading of the quantised
 *     BitLinear the pages cite).
 *
 * Parity pins for every function live in the CPU test suite (brute force on
 * tiny shapes against library routines, closed forms, invariants and a
 * hand-derived worked example); none is "parity unpinned".
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fno-fast-math
 * [-fopenmp].  Contraction of a*b+c into FMA is disabled so that the fp32
 * steps round exactly as written.
 */
#include "mmf_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

float orc_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

uint16_t orc_f64_to_bf16(double v) {
    /* bf16: 1 sign bit, 8 exponent bits (fp32 range), 8 significant bits
     * (7 stored).  Round |v| to the nearest multiple of the bf16 quantum at
     * its binade, ties to even, then read the bits off the exact fp32 value. */
    if (isnan(v)) return (uint16_t)0x7FC0;
    const int neg = signbit(v) ? 1 : 0;
    double a = fabs(v);
    double r;
    if (a == 0.0) {
        r = 0.0;
    } else if (a < ldexp(1.0, -126)) {
        /* subnormal range: fixed quantum 2^-133 */
        r = nearbyint(ldexp(a, 133));
        r = ldexp(r, -133);
    } else {
        int e;
        double m = frexp(a, &e);              /* a = m * 2^e, m in [0.5, 1) */
        double s = nearbyint(ldexp(m, 8));   /* 8 significant bits, ties even */
        r = ldexp(s, e - 8);
    }
    uint16_t out;
    if (r >= ldexp(1.0, 128)) {
        out = (uint16_t)0x7F80;               /* overflow to infinity */
    } else {
        float f = (float)r;                   /* exact: r has <= 8 significant bits */
        uint32_t u;
        memcpy(&u, &f, sizeof u);
        out = (uint16_t)(u >> 16);
    }
    return (uint16_t)(out | (neg ? 0x8000u : 0u));
}

void orc_absmean_ternary(const float* W, int64_t N, int64_t K, float eps_w,
                         int8_t* wt, float* beta) {
    const int64_t n = N * K;
    /* beta = mean |W|: sum in fp64, divide in fp64, round once to fp32. */
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i) s += fabs((double)W[i]);
    const float b = (n > 0) ? (float)(s / (double)n) : 0.0f;
    /* Divide (not multiply) by beta + eps_w, then RoundClip to {-1, 0, +1}.
     * The division and the rounding are fp32: this decides the code. */
    const float d = b + eps_w;
    for (int64_t i = 0; i < n; ++i) {
        const float t = W[i] / d;
        const float r = rintf(t);
        int8_t c;
        if (r > 1.0f) c = 1;
        else if (r < -1.0f) c = -1;
        else c = (int8_t)r;
        wt[i] = c;
    }
    *beta = b;
}

void orc_encode_packed(const int8_t* wt, int64_t N, int64_t K, uint32_t* packed) {
    const int64_t words = K / 16;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < words; ++j) {
            uint32_t w = 0;
            for (int i = 0; i < 16; ++i) {
                const int8_t t = wt[n * K + 16 * j + i];
                const uint32_t code = (uint32_t)(t + 1);   /* -1->0, 0->1, +1->2 */
                const int shift = 8 * (i % 4) + 2 * (i / 4);
                w |= code << shift;
            }
            packed[n * words + j] = w;
        }
    }
}

int64_t orc_decode_packed(const uint32_t* packed, int64_t N, int64_t K, int8_t* wt) {
    const int64_t words = K / 16;
    int64_t bad = 0;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < words; ++j) {
            const uint32_t w = packed[n * words + j];
            for (int i = 0; i < 16; ++i) {
                const int shift = 8 * (i % 4) + 2 * (i / 4);
                const uint32_t code = (w >> shift) & 3u;
                int8_t t;
                if (code == 3u) { ++bad; t = 0; }
                else t = (int8_t)((int)code - 1);
                wt[n * K + 16 * j + i] = t;
            }
        }
    }
    return bad;
}

void orc_rmsnorm_quant(const uint16_t* x, const float* gamma, float eps,
                       int64_t M, int64_t K, int8_t* q, float* absmax) {
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* xm = x + m * K;
        /* mean of squares: the bf16 values are exact in fp64, so are their
         * squares; sum and quotient in fp64, rounded once to fp32. */
        double s2 = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double v = (double)orc_bf16_to_f32(xm[k]);
            s2 += v * v;
        }
        const float ms = (float)(s2 / (double)K);
        const float inv = 1.0f / sqrtf(ms + eps);
        /* normalised, gained activations and their absolute maximum */
        float a = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            const float r = (orc_bf16_to_f32(xm[k]) * inv) * gamma[k];
            const float ar = fabsf(r);
            if (ar > a) a = ar;
        }
        if (a < 1e-5f) a = 1e-5f;
        const float s = 127.0f / a;
        for (int64_t k = 0; k < K; ++k) {
            const float r = (orc_bf16_to_f32(xm[k]) * inv) * gamma[k];
            const float t = rintf(r * s);
            int c;
            if (t > 127.0f) c = 127;
            else if (t < -127.0f) c = -127;
            else c = (int)t;
            q[m * K + k] = (int8_t)c;
        }
        absmax[m] = a;
    }
}

void orc_ternary_acc(const int8_t* q, const int8_t* wt, int64_t M, int64_t K,
                     int64_t N, int32_t* acc) {
#ifdef _OPENMP
#pragma omp parallel for collapse(2) schedule(static)
#endif
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            const int8_t* qm = q + m * K;
            const int8_t* wn = wt + n * K;
            int32_t s = 0;
            for (int64_t k = 0; k < K; ++k) {
                if (wn[k] == 1) s += qm[k];        /* +1: add      */
                else if (wn[k] == -1) s -= qm[k];  /* -1: subtract */
                /* 0: nothing */
            }
            acc[m * N + n] = s;
        }
    }
}

void orc_rescale(const int32_t* acc, const float* absmax, float beta,
                 int64_t M, int64_t N, uint16_t* y) {
    for (int64_t m = 0; m < M; ++m) {
        const double deq = ((double)absmax[m] / 127.0) * (double)beta;
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = orc_f64_to_bf16((double)acc[m * N + n] * deq);
    }
}

void orc_glu_gate(const uint16_t* g, const uint16_t* u, int64_t n, uint16_t* p) {
    for (int64_t i = 0; i < n; ++i) {
        const float gv = orc_bf16_to_f32(g[i]);
        const float uv = orc_bf16_to_f32(u[i]);
        const float sig = 1.0f / (1.0f + expf(-gv));
        const float silu = gv * sig;
        p[i] = orc_f64_to_bf16((double)(silu * uv));
    }
}

static float orc_sigmoid(float v) { return 1.0f / (1.0f + expf(-v)); }

void orc_mlgru_scan(const uint16_t* f_pre, const uint16_t* c_pre, const uint16_t* g_pre,
                    const float* h0, int64_t B, int64_t T, int64_t D, uint16_t* o, float* h_last) {
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t k = 0; k < D; ++k) {
            float h = h0 ? h0[b * D + k] : 0.0f;
            for (int64_t t = 0; t < T; ++t) {
                const int64_t i = (b * T + t) * D + k;
                const float f = orc_sigmoid(orc_bf16_to_f32(f_pre[i]));
                const float cv = orc_bf16_to_f32(c_pre[i]);
                const float c = cv * orc_sigmoid(cv);
                const float g = orc_sigmoid(orc_bf16_to_f32(g_pre[i]));
                h = f * h + (1.0f - f) * c;
                o[i] = orc_f64_to_bf16((double)(g * h));
            }
            h_last[b * D + k] = h;
        }
    }
}

int orc_bitlinear_bwd(const uint16_t* dy, const uint16_t* x, const float* gamma, float eps,
                      const int8_t* wt, float beta, int64_t M, int64_t K, int64_t N,
                      uint16_t* dx, float* dgamma, float* dW) {
    int8_t* q = (int8_t*)malloc((size_t)(M * K > 0 ? M * K : 1));
    float* a = (float*)malloc(sizeof(float) * (size_t)(M > 0 ? M : 1));
    double* dr = (double*)malloc(sizeof(double) * (size_t)(M * K > 0 ? M * K : 1));
    double* dg = (double*)calloc((size_t)(K > 0 ? K : 1), sizeof(double));
    if (!q || !a || !dr || !dg) {
        free(q);
        free(a);
        free(dr);
        free(dg);
        return -1;
    }
    orc_rmsnorm_quant(x, gamma, eps, M, K, q, a);
    /* dr = dy . W_q */
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0;
            for (int64_t n = 0; n < N; ++n) s += (double)orc_bf16_to_f32(dy[m * N + n]) * (double)wt[n * K + k];
            dr[m * K + k] = s * (double)beta;
        }
    /* dW = dy^T . x_q */
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0;
            for (int64_t m = 0; m < M; ++m)
                s += (double)orc_bf16_to_f32(dy[m * N + n]) * ((double)q[m * K + k] * ((double)a[m] / 127.0));
            dW[n * K + k] = (float)s;
        }
    /* RMSNorm backward */
    for (int64_t m = 0; m < M; ++m) {
        double s2 = 0.0, dot = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double xv = (double)orc_bf16_to_f32(x[m * K + k]);
            s2 += xv * xv;
            dot += (double)gamma[k] * dr[m * K + k] * xv;
        }
        const double inv = 1.0 / sqrt(s2 / (double)K + (double)eps);
        for (int64_t k = 0; k < K; ++k) {
            const double xv = (double)orc_bf16_to_f32(x[m * K + k]);
            const double g = inv * (double)gamma[k] * dr[m * K + k] - xv * inv * inv * inv * dot / (double)K;
            dx[m * K + k] = orc_f64_to_bf16(g);
            dg[k] += dr[m * K + k] * xv * inv;
        }
    }
    for (int64_t k = 0; k < K; ++k) dgamma[k] = (float)dg[k];
    free(q);
    free(a);
    free(dr);
    free(dg);
    return 0;
}

int orc_bitlinear(const uint16_t* x, const float* gamma, float eps,
                  const float* W, float eps_w, int64_t M, int64_t K, int64_t N,
                  uint16_t* y, float* beta_out) {
    int8_t* wt = (int8_t*)malloc((size_t)(N * K > 0 ? N * K : 1));
    int8_t* q = (int8_t*)malloc((size_t)(M * K > 0 ? M * K : 1));
    float* a = (float*)malloc(sizeof(float) * (size_t)(M > 0 ? M : 1));
    int32_t* acc = (int32_t*)malloc(sizeof(int32_t) * (size_t)(M * N > 0 ? M * N : 1));
    int rc = 0;
    if (!wt || !q || !a || !acc) {
        rc = -1;
    } else {
        float beta;
        orc_absmean_ternary(W, N, K, eps_w, wt, &beta);
        orc_rmsnorm_quant(x, gamma, eps, M, K, q, a);
        orc_ternary_acc(q, wt, M, K, N, acc);
        orc_rescale(acc, a, beta, M, N, y);
        if (beta_out) *beta_out = beta;
    }
    free(wt);
    free(q);
    free(a);
    free(acc);
    return rc;
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
