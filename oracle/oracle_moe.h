/*
 * oracle_moe.h -- CPU oracle for the MoE feed-forward layer with MXFP4 experts.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load or call this library.  It shares no
 * code, header, table or constant with the CUDA library, and the product path
 * never routes through it.
 *
 * Everything is a plain, slow restatement in double precision of what the
 * layer computes, following the page "GPT-OSS-20B : Architecture MoE & Résumé
 * du Model Card":
 *   §3.1 Le Routeur       scores = W_router . h, top-k selection, softmax over
 *                         the selected scores so the k weights sum to 1;
 *   §3.2 Les Experts      SwiGLU expert (Swish(x W_gate) (.) (x W_up)) W_down
 *                         with Swish(x) = x sigma(x);
 *   §2.1 Qu'est-ce qu'un modèle MoE ?  the k expert outputs are aggregated
 *                         with different weights;
 *   §4 Quantification MXFP4   4.25 bits per parameter: blocks of 32 FP4
 *                         (E2M1) codes that share one 8-bit power-of-two
 *                         (E8M0) scale -- the Microscaling format of Darvish
 *                         Rouhani et al. 2023, which that page cites;
 * and, from the page "GPT-OSS vs Qwen3 : comparaison détaillée", Adoption de
 * RMSNorm: the block's input is normalised by its root mean square.
 *
 * Weight layout used by every function here (the "canonical" layout): for a
 * matrix applied as y = x . W with contraction length K and N outputs, row n
 * (n < N) holds the K weights that feed output n.  codes: [N][K/2] bytes, the
 * element with even k in the low nibble; scales: [N][K/32] E8M0 bytes.
 */
#ifndef ORACLE_MOE_H
#define ORACLE_MOE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Value of one E2M1 code (bit 3 sign, bits 2..1 exponent, bit 0 mantissa). */
double oracle_e2m1_decode(uint32_t code);

/* 2^(s-127) for an E8M0 scale byte s (255, the NaN encoding, returns NaN). */
double oracle_e8m0_decode(uint32_t s);

/* Quantise `rows` vectors of length K (K % 32 == 0) to MXFP4.
 * Element (n, k) is read from w[n*s_row + k*s_k].  Writes codes [rows][K/2]
 * and scales [rows][K/32]. */
void oracle_mxfp4_quantize(const float* w, int64_t rows, int64_t K,
                           int64_t s_row, int64_t s_k,
                           uint8_t* codes, uint8_t* scales);

/* Dequantise rows [row0, row0+nrows) of a canonical MXFP4 matrix to double
 * (out: [nrows][K]). */
void oracle_mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales,
                             int64_t K, int64_t row0, int64_t nrows, double* out);

/* Swish(z) = z * sigma(z), sigma(z) = 1/(1+exp(-z)). */
double oracle_swish(double z);

/* Router for T tokens: logits[t][e] = sum_i x[t][i] * wr[e][i] + bias[e]
 * (bias may be NULL); idx[t][j] = the k largest logits in descending order,
 * ties to the lower expert index; w[t][j] = softmax over the k selected
 * logits; counts[e] = number of (t, j) with idx[t][j] == e.
 * Any of logits / idx / w / counts may be NULL. */
void oracle_router(const double* x, int64_t T, int64_t d,
                   const double* wr, int64_t E, const double* bias, int32_t k,
                   double* logits, int32_t* idx, double* w, int64_t* counts);

/* One SwiGLU expert applied to one row x[d_model]:
 *   g = x . W_gate, u = x . W_up (length d_ff), h = Swish(g) * u,
 *   out = h . W_down (length d_model).
 * gate/up: canonical [d_ff][d_model/2] codes, [d_ff][d_model/32] scales;
 * down: canonical [d_model][d_ff/2] codes, [d_model][d_ff/32] scales.
 * h_out (length d_ff) may be NULL. */
void oracle_expert(const double* x, int64_t d_model, int64_t d_ff,
                   const uint8_t* g_codes, const uint8_t* g_scales,
                   const uint8_t* u_codes, const uint8_t* u_scales,
                   const uint8_t* d_codes, const uint8_t* d_scales,
                   double* out, double* h_out);

/* Layer output for a list of tokens.
 * x: [T][d_model]; idx/w: [T][k] from oracle_router; expert weights stored
 * expert-major: gate codes [E][d_ff][d_model/2], scales [E][d_ff][d_model/32],
 * same for up; down codes [E][d_model][d_ff/2], scales [E][d_model][d_ff/32].
 * For each of the n_tok tokens t = tokens[i] (tokens == NULL means 0..n_tok-1):
 *   y[i][:] = sum_j w[t][j] * expert_{idx[t][j]}(x[t]).
 * nthreads > 1 splits the token list over POSIX threads (rows are
 * independent, so the result does not depend on the thread count). */
void oracle_moe_forward(const double* x, int64_t d_model, int64_t d_ff, int64_t E,
                        int32_t k, const int32_t* idx, const double* w,
                        const uint8_t* g_codes, const uint8_t* g_scales,
                        const uint8_t* u_codes, const uint8_t* u_scales,
                        const uint8_t* d_codes, const uint8_t* d_scales,
                        const int64_t* tokens, int64_t n_tok, double* y,
                        int32_t nthreads);

/* RMSNorm of T tokens (page "GPT-OSS vs Qwen3 : comparaison détaillée",
 * Adoption de RMSNorm: normalise by the root mean square instead of LayerNorm's
 * mean and variance):
 *   out[t][i] = x[t][i] / sqrt(mean_j x[t][j]^2 + eps) * gamma[i]
 * (gamma == NULL means all ones).  x and out may alias only if equal. */
void oracle_rmsnorm(const double* x, int64_t T, int64_t d, const double* gamma,
                    double eps, double* out);

#ifdef __cplusplus
}
#endif
#endif
