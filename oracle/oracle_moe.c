/*
 * oracle_moe.c -- plain double-precision CPU oracle for the MoE layer with
 * MXFP4 experts.  TEST INFRASTRUCTURE ONLY (see oracle_moe.h): nothing in the
 * product path links or calls this file.
 *
 * Sources restated here (page "GPT-OSS-20B : Architecture MoE & Résumé du
 * Model Card"): §3.1 Le Routeur (linear scores, top-k, softmax over the
 * selected scores summing to 1), §3.2 Les Experts (SwiGLU with Swish(x) =
 * x sigma(x) and three matrices W_gate, W_up, W_down), §2.1 (weighted
 * aggregation of the k expert outputs), §4 Quantification MXFP4 (4.25 bits
 * per parameter; Microscaling format of Darvish Rouhani et al. 2023: blocks of
 * 32 E2M1 elements sharing one E8M0 scale).  Page "GPT-OSS vs Qwen3 :
 * comparaison détaillée", Adoption de RMSNorm: the normalisation next to the
 * block divides by the root mean square of the token instead of using the
 * mean and variance.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - block scale exponent: floor(log2(max|w|)) - 2, clamped to [-127, 127];
 *    2 is the exponent of the largest E2M1 magnitude (6 = 1.5 * 2^2);
 *  - element rounding: nearest E2M1 magnitude, ties to the even code,
 *    magnitudes above 6 saturate to 6, sign bit kept (so -0 is code 8);
 *  - an all-zero block gets scale 2^0 (byte 127) and zero codes;
 *  - top-k ties go to the lower expert index; k outputs in descending order;
 *  - no expert biases, no clamping, Swish with beta = 1.
 */
#include "oracle_moe.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* E2M1 magnitudes by the low three code bits (exponent bits e1 e0, mantissa m):
 * e = 0 gives the subnormal values 0 and 0.5; otherwise (1 + m/2) * 2^(e-1). */
static double e2m1_magnitude(uint32_t c3) {
    uint32_t e = (c3 >> 1) & 3u, m = c3 & 1u;
    if (e == 0) return 0.5 * (double)m;
    return (1.0 + 0.5 * (double)m) * ldexp(1.0, (int)e - 1);
}

double oracle_e2m1_decode(uint32_t code) {
    double mag = e2m1_magnitude(code & 7u);
    return (code & 8u) ? -mag : mag;
}

double oracle_e8m0_decode(uint32_t s) {
    if ((s & 0xFFu) == 255u) return NAN;
    return ldexp(1.0, (int)(s & 0xFFu) - 127);
}

/* Lookup tables filled once from the decode functions above: the 16 E2M1 code
 * values and the 256 E8M0 scale values (tables only avoid recomputing them). */
static double g_code_value[16];
static double g_scale_value[256];
static pthread_once_t g_tables_once = PTHREAD_ONCE_INIT;
static void fill_tables(void) {
    for (uint32_t c = 0; c < 16; ++c) g_code_value[c] = oracle_e2m1_decode(c);
    for (uint32_t s = 0; s < 256; ++s) g_scale_value[s] = oracle_e8m0_decode(s);
}
static void tables(void) { pthread_once(&g_tables_once, fill_tables); }

/* Nearest E2M1 magnitude code for a >= 0; equal distances go to the even code. */
static uint32_t e2m1_round_magnitude(double a) {
    uint32_t best = 0;
    double best_d = fabs(a - g_code_value[0]);
    for (uint32_t c = 1; c < 8; ++c) {
        double dd = fabs(a - g_code_value[c]);
        if (dd < best_d || (dd == best_d && (c & 1u) == 0 && (best & 1u) == 1)) {
            best = c;
            best_d = dd;
        }
    }
    return best;
}

void oracle_mxfp4_quantize(const float* w, int64_t rows, int64_t K,
                           int64_t s_row, int64_t s_k,
                           uint8_t* codes, uint8_t* scales) {
    const int64_t nb = K / 32;
    tables();
    for (int64_t n = 0; n < rows; ++n) {
        for (int64_t b = 0; b < nb; ++b) {
            double v[32];
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                v[i] = (double)w[n * s_row + (b * 32 + i) * s_k];
                if (fabs(v[i]) > amax) amax = fabs(v[i]);
            }
            uint8_t* cb = codes + n * (K / 2) + b * 16;
            if (amax == 0.0) {
                scales[n * nb + b] = 127;
                memset(cb, 0, 16);
                continue;
            }
            int ex;
            frexp(amax, &ex);            /* amax = f * 2^ex, 0.5 <= f < 1 */
            int X = ex - 1;              /* floor(log2(amax)), exact */
            int e = X - 2;
            if (e < -127) e = -127;
            if (e > 127) e = 127;
            scales[n * nb + b] = (uint8_t)(e + 127);
            for (int i = 0; i < 32; ++i) {
                double s = ldexp(v[i], -e); /* exact power-of-two rescale */
                uint32_t c = e2m1_round_magnitude(fabs(s));
                if (signbit(v[i])) c |= 8u;
                if (i & 1) cb[i / 2] |= (uint8_t)(c << 4);
                else cb[i / 2] = (uint8_t)c;
            }
        }
    }
}

static inline double mx_value(const uint8_t* codes, const uint8_t* scales,
                              int64_t K, int64_t n, int64_t k) {
    uint8_t byte = codes[n * (K / 2) + k / 2];
    uint32_t c = (k & 1) ? (uint32_t)(byte >> 4) : (uint32_t)(byte & 15u);
    return g_code_value[c] * g_scale_value[scales[n * (K / 32) + k / 32]];
}

void oracle_mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales,
                             int64_t K, int64_t row0, int64_t nrows, double* out) {
    tables();
    for (int64_t r = 0; r < nrows; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = mx_value(codes, scales, K, row0 + r, k);
}

double oracle_swish(double z) { return z / (1.0 + exp(-z)); }

void oracle_router(const double* x, int64_t T, int64_t d,
                   const double* wr, int64_t E, const double* bias, int32_t k,
                   double* logits, int32_t* idx, double* w, int64_t* counts) {
    double* s = (double*)malloc(sizeof(double) * (size_t)E);
    int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)(k > 0 ? k : 1));
    char* taken = (char*)malloc((size_t)E);
    if (counts)
        for (int64_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t t = 0; t < T; ++t) {
        /* scores = W_router . h */
        for (int64_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t i = 0; i < d; ++i) acc += x[t * d + i] * wr[e * d + i];
            if (bias) acc += bias[e];
            s[e] = acc;
            if (logits) logits[t * E + e] = acc;
        }
        /* top-k: repeatedly take the largest remaining score (lower index on ties) */
        memset(taken, 0, (size_t)E);
        for (int32_t j = 0; j < k; ++j) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || s[e] > s[best]) best = e;
            }
            taken[best] = 1;
            sel[j] = (int32_t)best;
        }
        /* softmax over the selected scores */
        double smax = s[sel[0]];
        for (int32_t j = 1; j < k; ++j)
            if (s[sel[j]] > smax) smax = s[sel[j]];
        double den = 0.0;
        for (int32_t j = 0; j < k; ++j) den += exp(s[sel[j]] - smax);
        for (int32_t j = 0; j < k; ++j) {
            if (idx) idx[t * k + j] = sel[j];
            if (w) w[t * k + j] = exp(s[sel[j]] - smax) / den;
            if (counts) counts[sel[j]] += 1;
        }
    }
    free(s);
    free(sel);
    free(taken);
}

void oracle_expert(const double* x, int64_t d_model, int64_t d_ff,
                   const uint8_t* g_codes, const uint8_t* g_scales,
                   const uint8_t* u_codes, const uint8_t* u_scales,
                   const uint8_t* d_codes, const uint8_t* d_scales,
                   double* out, double* h_out) {
    tables();
    double* h = (double*)malloc(sizeof(double) * (size_t)d_ff);
    for (int64_t f = 0; f < d_ff; ++f) {
        double g = 0.0, u = 0.0;
        for (int64_t i = 0; i < d_model; ++i) {
            g += x[i] * mx_value(g_codes, g_scales, d_model, f, i);
            u += x[i] * mx_value(u_codes, u_scales, d_model, f, i);
        }
        h[f] = oracle_swish(g) * u;
        if (h_out) h_out[f] = h[f];
    }
    for (int64_t o = 0; o < d_model; ++o) {
        double acc = 0.0;
        for (int64_t f = 0; f < d_ff; ++f) acc += h[f] * mx_value(d_codes, d_scales, d_ff, o, f);
        out[o] = acc;
    }
    free(h);
}

typedef struct {
    const double* x;
    int64_t d_model, d_ff, E;
    int32_t k;
    const int32_t* idx;
    const double* w;
    const uint8_t *gc, *gs, *uc, *us, *dc, *ds;
    const int64_t* tokens;
    int64_t n_tok;
    double* y;
    int32_t tid, nthreads;
} fwd_job_t;

static void* fwd_worker(void* arg) {
    fwd_job_t* J = (fwd_job_t*)arg;
    const int64_t d = J->d_model, f = J->d_ff;
    const int64_t gc_sz = f * (d / 2), gs_sz = f * (d / 32);
    const int64_t dc_sz = d * (f / 2), ds_sz = d * (f / 32);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    for (int64_t i = J->tid; i < J->n_tok; i += J->nthreads) {
        int64_t t = J->tokens ? J->tokens[i] : i;
        double* yi = J->y + i * d;
        for (int64_t c = 0; c < d; ++c) yi[c] = 0.0;
        for (int32_t j = 0; j < J->k; ++j) {
            int64_t e = J->idx[t * J->k + j];
            oracle_expert(J->x + t * d, d, f,
                          J->gc + e * gc_sz, J->gs + e * gs_sz,
                          J->uc + e * gc_sz, J->us + e * gs_sz,
                          J->dc + e * dc_sz, J->ds + e * ds_sz, o, NULL);
            double wj = J->w[t * J->k + j];
            for (int64_t c = 0; c < d; ++c) yi[c] += wj * o[c];
        }
    }
    free(o);
    return NULL;
}

void oracle_moe_forward(const double* x, int64_t d_model, int64_t d_ff, int64_t E,
                        int32_t k, const int32_t* idx, const double* w,
                        const uint8_t* g_codes, const uint8_t* g_scales,
                        const uint8_t* u_codes, const uint8_t* u_scales,
                        const uint8_t* d_codes, const uint8_t* d_scales,
                        const int64_t* tokens, int64_t n_tok, double* y,
                        int32_t nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    fwd_job_t* jobs = (fwd_job_t*)malloc(sizeof(fwd_job_t) * (size_t)nthreads);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int32_t i = 0; i < nthreads; ++i) {
        fwd_job_t J = {x, d_model, d_ff, E, k, idx, w, g_codes, g_scales, u_codes,
                       u_scales, d_codes, d_scales, tokens, n_tok, y, i, nthreads};
        jobs[i] = J;
    }
    for (int32_t i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, fwd_worker, &jobs[i]);
    fwd_worker(&jobs[0]);
    for (int32_t i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(jobs);
    free(th);
}

void oracle_rmsnorm(const double* x, int64_t T, int64_t d, const double* gamma,
                    double eps, double* out) {
    for (int64_t t = 0; t < T; ++t) {
        /* root mean square of the token's d values (the mean, not the sum) */
        double ss = 0.0;
        for (int64_t i = 0; i < d; ++i) ss += x[t * d + i] * x[t * d + i];
        const double rms = sqrt(ss / (double)d + eps);
        for (int64_t i = 0; i < d; ++i) {
            const double g = gamma ? gamma[i] : 1.0;
            out[t * d + i] = x[t * d + i] / rms * g;
        }
    }
}
