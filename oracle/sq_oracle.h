/*
 * sq_oracle.h -- CPU oracle for the SmoothQuant W8A8 INT8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, obviously-correct CPU
 * restatement of what the layer computes.  Only the test suite, the smoke
 * check of the package entry file and the CPU-baseline leg of the benchmark
 * may load it.  It shares no code, header, table or helper with the CUDA
 * library, and the CUDA library never calls it.
 *
 * Sources, by page title and section:
 *  - "Qwen3.8-27B - SmoothQuant + activation-aware GPTQ, W8A8 INT8 (v3)",
 *    section "Recipe", items 1-2: SmoothQuant folds (1/s into the
 *    preceding norm, s into the next linear), smoothing scales capped at 16,
 *    INT8 per-channel symmetric weights, INT8 per-token dynamic activations;
 *    W8A16 (INT8 per-channel weights, BF16 activations) for down_proj.
 *  - "Qwen3.8-27B - FP8 block + AWQ", section "Recipe", item 1: the fold is
 *    function preserving and the ratio to the original weights is a
 *    separable per-row x per-column scale.
 *  - "Qwen3.8-27B-INT8-W8A8", section "Quantization": symmetric INT8 weights
 *    per output channel, INT8 dynamic per-token activations.
 *  - "Qwen3.8-27B-GPTQ-INT8-W8A8-GS128", section "Quantization details" and
 *    the paragraph "Why group_size 128": 8 bits, symmetric, one weight scale
 *    per 128-wide K block, INT8 x INT8 compute with the inputs quantised
 *    dynamically.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 * round-to-nearest-even; scale = amax/127 and multiplier 127/amax, both fp32
 * IEEE divisions; codes clamped to [-127, 127] (symmetric, -128 never used);
 * an all-zero row gets scale 0 and codes 0; the per-channel epilogue is
 * (f32(acc) * s_tok) * s_ch with two fp32 roundings then BF16 RNE; the gs128
 * accumulation is fmaf(f32(P_kb), s_blk, acc) over blocks in ascending order,
 * then * s_tok; W8A16 is the exact (fp64) sum times s_ch, rounded once to BF16.
 *
 * Layouts: row-major, contiguous.  X [M,K] bf16 (as uint16 bits), W [N,K]
 * bf16, q_a [M,K] int8, q_w [N,K] int8, s_tok [M] f32, s_ch [N] f32,
 * s_blk [N, K/128] f32, y [M,N] bf16 bits, acc [M,N] int32.
 * Functions return 0 on success and a negative number on bad arguments.
 */
#ifndef SQ_ORACLE_H
#define SQ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Scalar conversions, exported so the tests can pin them. */
uint16_t oracle_f32_to_bf16(float f);            /* RNE, NaN -> quiet NaN */
uint16_t oracle_f64_to_bf16(double d);           /* RNE, one rounding     */
float    oracle_bf16_to_f32(uint16_t h);

/* Smoothing factors: s_j = clamp(sqrt(max_m|X[m,j]|) / sqrt(max_n|W[n,j]|),
 * floor, cap) in fp64 (alpha = 1/2); s_out[j] = f32(s_j),
 * inv_s_out[j] = f32(1 / s_out[j]).  A column whose X and W maxima are both
 * zero gets s = 1; one with max|W| = 0 only gets s = cap. */
int oracle_smooth_factors(const uint16_t* x, int64_t M, int64_t K,
                          const uint16_t* w, int64_t N, double cap, double floor_,
                          float* s_out, float* inv_s_out);

/* Folded weight W'[n,k] = f32(W[n,k] * s[k]) (s may be NULL: W' = W). */
int oracle_fold_weight(const uint16_t* w, int64_t N, int64_t K, const float* s,
                       float* w_folded);

/* Symmetric INT8 weight quantisation of W' = fold(W, s).
 * group == 0: one scale per output row; group == 128: one per (row, K block).
 * scales has N (group 0) or N*K/group (row-major) entries. */
int oracle_quant_weight(const uint16_t* w, int64_t N, int64_t K, const float* s,
                        int64_t group, int8_t* q, float* scales);

/* Per-token dynamic quantisation with the 1/s fold:
 * x' = f32(x) * inv_s[k]; amax = max|x'|; s_tok = amax/127;
 * q = clamp(rint(x' * (127/amax)), -127, 127).  inv_s may be NULL (= 1). */
int oracle_quant_per_token(const uint16_t* x, int64_t M, int64_t K,
                           const float* inv_s, int8_t* q, float* s_tok);

/* The rows computed by the GEMM functions: rows == NULL means all M rows
 * (nrows == M); otherwise output row r is input row rows[r].  Outputs have
 * nrows rows. */
int oracle_mm_i32(const int8_t* q_a, const int8_t* q_w, int64_t M, int64_t N,
                  int64_t K, const int64_t* rows, int64_t nrows, int32_t* acc);

int oracle_epilogue_ch(const int32_t* acc, const float* s_tok, const float* s_ch,
                       int64_t nrows, int64_t N, uint16_t* y);

int oracle_w8a8_scaled_mm(const int8_t* q_a, const float* s_tok, const int8_t* q_w,
                          const float* s_ch, int64_t M, int64_t N, int64_t K,
                          const int64_t* rows, int64_t nrows, uint16_t* y);

int oracle_gs128_mm(const int8_t* q_a, const float* s_tok, const int8_t* q_w,
                    const float* s_blk, int64_t M, int64_t N, int64_t K,
                    const int64_t* rows, int64_t nrows, uint16_t* y);

/* W8A16: y = bf16(s_ch[n] * sum_k f32(x[m,k]) * q_w[n,k]), sum in fp64.
 * Also returns, if abs_out != NULL, sum_k |x * q| * s_ch per output (fp64),
 * which bounds the rounding error of any fp32 accumulation order. */
int oracle_w8a16_mm(const uint16_t* x, const int8_t* q_w, const float* s_ch,
                    int64_t M, int64_t N, int64_t K, const int64_t* rows,
                    int64_t nrows, uint16_t* y, double* abs_out);

/* ---- Next rows of the layer ------------------------------------------
 * Sources (page title, section):
 *  - "Qwen3.8-27B - SmoothQuant + activation-aware GPTQ, W8A8 INT8 (v3)",
 *    "Recipe" item 1 and "Qwen3.8-27B - FP8 block + AWQ", "Recipe" item 1:
 *    the smoothing factor 1/s is absorbed into the (zero-centred) norm that
 *    precedes the linear layer.
 *  - "Qwen3.8-27B-GPTQ-INT8-W8A8-GS128", "Serving (vLLM, gfx908 fork)":
 *    fused RMSNorm with per-group INT8 quantised output, W8A8 INT8 GEMMs
 *    with one weight scale per 128-wide K block at every M.
 *  - "lued/Qwen3.8-27B-INT8-W8A16-MTP", "Why W8A16 on Ampere": weight-only
 *    kernels reconstruct 16-bit weights; eight integer bits with group-wise
 *    scaling.
 *  - "Qwen3.8-27B - FP8 block + AWQ", "Recipe" item 2 and the note below it:
 *    FP8 weights with one scale per [128, 128] block, activations quantised
 *    dynamically per group, every quantised dimension divisible by 128.
 *
 * Readings where the pages are silent (listed in the design notes):
 *  RMSNorm: ss = sum_k f32(h_k)^2 computed exactly, rounded once to fp32
 *  (RNE); ms = ss / K, r = 1 / sqrt(ms + eps), each an IEEE fp32 operation;
 *  x'_k = (f32(h_k) * r) * gamma_k with two fp32 roundings; gamma is the norm
 *  weight with 1/s folded in, gamma_k = f32(g_k * inv_s_k), g_k = 1 + w_k
 *  (fp32) for a zero-centred norm, else w_k; eps > 0.  Then the quantisation
 *  of quant_per_token, over the whole row (group == K) or per 128 columns.
 *  Per-group activations: the quantisation of quant_per_token applied to
 *  each 128-wide block of a row; GEMM promotion
 *  acc = fmaf(f32(P_kb), f32(s_a[m,kb] * s_blk[n,kb]), acc) in ascending kb,
 *  y = bf16(acc).
 *  Group-wise W8A16: codes and scales as the gs128 weight quantisation;
 *  reconstructed weight w_hat = bf16(f32(q * s_grp)) (two roundings, RNE);
 *  y = bf16(sum_k x * w_hat) with the sum taken exactly (fp64).
 *  FP8: OCP E4M3 (bias 7, max 448, no infinities), round-half-even with
 *  saturation to +-448; scale = amax / 448, code = e4m3(v * (448 / amax))
 *  (fp32 product); amax == 0 gives scale 0 and zero codes.  GEMM:
 *  y = bf16(sum_kb P_kb * f32(s_a[m,kb] * s_w[n/128,kb])) with P_kb the
 *  exact block dot product of the decoded codes and the outer sum exact
 *  (fp64); the GPU accumulates in fp32, so it is compared within a bound.
 */

/* Zero-centred (or plain) norm weight with 1/s folded in:
 * gamma[k] = f32(g_k * inv_s[k]), g_k = 1 + f32(w[k]) if zero_centered else
 * f32(w[k]); inv_s may be NULL (= 1).  w is bf16 [K]. */
int oracle_fold_norm_weight(const uint16_t* w, int64_t K, int zero_centered,
                            const float* inv_s, float* gamma);

/* Exact sum of squares of n bf16 values, rounded once to fp32 (RNE). */
float oracle_sumsq_f32(const uint16_t* h, int64_t n);

/* Fused RMSNorm + fold + dynamic INT8 quantisation of h bf16 [M,K].
 * group == K: one scale per row (scales [M]); group == 128: one per
 * 128-wide block (scales [M, K/128]).  r_out (fp32 [M], optional) receives
 * r = 1/sqrt(ms + eps).  r_in (optional, test use): take r from it instead
 * of computing it, so the steps after the reduction can be checked alone. */
int oracle_rmsnorm_quant(const uint16_t* h, int64_t M, int64_t K, const float* gamma,
                         float eps, int64_t group, const float* r_in, int8_t* q,
                         float* scales, float* r_out);

/* Per-group (1 x 128) dynamic INT8 quantisation of x bf16 [M,K] with the
 * 1/s fold (inv_s may be NULL): s_a fp32 [M, K/128]. */
int oracle_quant_per_group(const uint16_t* x, int64_t M, int64_t K, const float* inv_s,
                           int8_t* q, float* s_a);

/* Per-group activations x gs128 weights:
 * y = bf16(acc), acc = fmaf(f32(P_kb), f32(s_a[m,kb] * s_blk[n,kb]), acc). */
int oracle_pg128_mm(const int8_t* q_a, const float* s_a, const int8_t* q_w,
                    const float* s_blk, int64_t M, int64_t N, int64_t K,
                    const int64_t* rows, int64_t nrows, uint16_t* y);

/* Reconstructed group-wise W8A16 weight: w_hat[n,k] = bf16(f32(q * s_grp[n,k/128])). */
int oracle_dequant_weight_group(const int8_t* q_w, const float* s_grp, int64_t N, int64_t K,
                                uint16_t* w_hat);

/* Group-wise W8A16: y = bf16(sum_k f32(x) * w_hat) (exact sum, one rounding);
 * abs_out (optional) = sum_k |x * w_hat| per output. */
int oracle_w8a16_group_mm(const uint16_t* x, const int8_t* q_w, const float* s_grp,
                          int64_t M, int64_t N, int64_t K, const int64_t* rows,
                          int64_t nrows, uint16_t* y, double* abs_out);

/* OCP E4M3 conversions (RNE, saturating to +-448; NaN stays NaN). */
uint8_t oracle_f32_to_e4m3(float v);
float   oracle_e4m3_to_f32(uint8_t b);

/* FP8 per-group (1 x 128) activations: q e4m3 [M,K], s_a fp32 [M, K/128]. */
int oracle_quant_fp8_per_group(const uint16_t* x, int64_t M, int64_t K, const float* inv_s,
                               uint8_t* q, float* s_a);

/* FP8 block weights: one scale per [128, 128] block of the folded weight
 * f32(w) * smooth[k] (smooth may be NULL); N % 128 == 0, K % 128 == 0;
 * q e4m3 [N,K], s_w fp32 [N/128, K/128]. */
int oracle_quant_fp8_block(const uint16_t* w, int64_t N, int64_t K, const float* smooth,
                           uint8_t* q, float* s_w);

/* FP8 block GEMM: y = bf16(sum_kb P_kb * f32(s_a[m,kb] * s_w[n/128,kb])),
 * P_kb the exact dot product of block kb, the outer sum exact (fp64).
 * abs_out (optional) = sum_kb |scale_kb| * sum_k |a * w| per output. */
int oracle_fp8_block_mm(const uint8_t* q_a, const float* s_a, const uint8_t* q_w,
                        const float* s_w, int64_t M, int64_t N, int64_t K,
                        const int64_t* rows, int64_t nrows, uint16_t* y, double* abs_out);

/* Worker threads the oracle uses (set before a call; 0 = hardware count). */
void oracle_set_threads(int n);
int  oracle_get_threads(void);

#ifdef __cplusplus
}
#endif
#endif
