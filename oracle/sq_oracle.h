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

/* Worker threads the oracle uses (set before a call; 0 = hardware count). */
void oracle_set_threads(int n);
int  oracle_get_threads(void);

#ifdef __cplusplus
}
#endif
#endif
