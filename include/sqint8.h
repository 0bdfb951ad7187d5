/*
 * sqint8.h -- C ABI of the B200 (sm_100a) SmoothQuant W8A8 INT8 linear layer.
 *
 * Every call is asynchronous on the caller's CUDA stream (passed as a
 * cudaStream_t cast to void*; NULL is the legacy default stream).  The
 * library never allocates device memory and never synchronises: the caller
 * owns every buffer (device pointers, row-major, contiguous, 16-byte
 * aligned) and the stream.  Errors are returned as sq_status; nothing aborts,
 * exits or traps.  A kernel wait that exceeds its time limit makes the kernel
 * return early and latch a device error word, read by sq_check_device_error.
 *
 * Shapes: M >= 0 tokens, N > 0 output channels with N % 16 == 0,
 * K > 0 input channels with K % 128 == 0 and K <= 131072 (so that
 * K * 127 * 127 fits in int32).  M == 0 is a no-op.
 *
 * Sources (page title, section):
 *  [P1] "Qwen3.8-27B - SmoothQuant + activation-aware GPTQ, W8A8 INT8 (v3)",
 *       "Recipe" items 1-2 and "Serving": SmoothQuant folds; INT8 per-channel
 *       symmetric weights with INT8 per-token dynamic activations (W8A8) on
 *       a scaled-mm kernel; INT8 per-channel weights with BF16 activations
 *       (W8A16) for down_proj on a weight-only dequant kernel.
 *  [P2] "lued/Qwen3.8-27B-INT8-W8A16-MTP", "Why W8A16 on Ampere": weight-only
 *       kernels reconstruct the weights for 16-bit GEMMs.
 *  [P3] "Qwen3.8-27B - FP8 block + AWQ", "Recipe" item 1: 1/s folds into the
 *       preceding op, s into the next linear's input dimension.
 *  [P4] "Qwen3.8-27B-INT8-W8A8", "Quantization": symmetric per-output-channel
 *       INT8 weights, dynamic per-token INT8 activations.
 *  [P5] "Qwen3.8-27B-GPTQ-INT8-W8A8-GS128", "Quantization details" and
 *       "Why group_size 128": one weight scale per 128-wide K block with INT8
 *       x INT8 compute and dynamically quantised inputs; "Serving (vLLM,
 *       gfx908 fork)": fused RMSNorm with per-group INT8 quantised output and
 *       W8A8 INT8 GEMMs at every M.
 *  [P3b] "Qwen3.8-27B - FP8 block + AWQ", "Recipe" item 2 and the note after
 *       it: FP8 weights with one scale per [128, 128] block, activations
 *       quantised dynamically per group, quantised dimensions divisible by 128.
 */
#ifndef SQINT8_H
#define SQINT8_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SQ_OK = 0,
  SQ_ERR_NULL = 1,        /* a required pointer is NULL                          */
  SQ_ERR_SHAPE = 2,       /* a size breaks the rules above                       */
  SQ_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned                    */
  SQ_ERR_WORKSPACE = 4,   /* workspace missing or smaller than sq_workspace_bytes */
  SQ_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed                   */
  SQ_ERR_TIMEOUT = 6      /* a kernel gave up a wait (sq_check_device_error)     */
} sq_status;

/* Operation ids for sq_workspace_bytes. */
enum { SQ_OP_W8A8 = 0, SQ_OP_GS128 = 1, SQ_OP_W8A16 = 2, SQ_OP_W8A8_I32 = 3,
       SQ_OP_PG128 = 4, SQ_OP_FP8BLK = 5, SQ_OP_W8A16_GROUP = 6 };

/* Per-token dynamic INT8 quantisation with the SmoothQuant 1/s fold [P1, P3, P4].
 * For each row m of x (BF16 [M,K]):  x'[k] = f32(x[m,k]) * inv_smooth[k]
 * (one fp32 rounding), amax = max_k |x'[k]|, s_tok[m] = amax / 127,
 * q_i8[m,k] = clamp(rint(x'[k] * (127 / amax)), -127, 127) with
 * round-half-even; an all-zero row gives s_tok = 0 and zero codes.
 * inv_smooth (fp32 [K]) may be NULL (no smoothing).
 * Outputs: q_i8 int8 [M,K], s_tok fp32 [M]. */
sq_status sq_quant_per_token(const void* x_bf16, const float* inv_smooth, int8_t* q_i8,
                             float* s_tok, int64_t M, int64_t K, void* stream);

/* W8A8 INT8 GEMM with the fused per-token x per-channel dequant epilogue
 * [P1 "Serving", P4]:  acc[m,n] = sum_k q_a[m,k] * q_w[n,k] (exact int32),
 * y[m,n] = bf16_rne((f32(acc) * s_tok[m]) * s_ch[n]).
 * q_a int8 [M,K], s_tok fp32 [M], q_w int8 [N,K] (nn.Linear layout, K-major),
 * s_ch fp32 [N], y_bf16 [M,N].  Small M (<= 32) uses a split-K schedule
 * whose partial sums live in the caller's workspace (size from
 * sq_workspace_bytes(SQ_OP_W8A8, ...); pass NULL/0 when it is 0).
 * Workspace rule for every operation: the first 64 KiB hold arrival
 * counters that must be zero before the workspace is first used; every call
 * that completes on the device leaves them zero, and nothing else is written
 * there, so one workspace may serve calls of any operation and size in
 * stream order.  Calls that may overlap on the device need separate
 * workspaces.  After SQ_ERR_TIMEOUT, zero the counters again. */
sq_status w8a8_scaled_mm(const int8_t* q_a, const float* s_tok, const int8_t* q_w,
                         const float* s_ch, void* y_bf16, int64_t M, int64_t N, int64_t K,
                         void* workspace, size_t ws_bytes, void* stream);

/* The whole W8A8 linear layer in one call [P1, P4]: sq_quant_per_token of x
 * into the caller's q_a (int8 [M,K]) and s_tok (fp32 [M]), then
 * w8a8_scaled_mm into y.  The GEMM is launched as a programmatic dependent of
 * the quantisation kernel: it may start, allocate tensor memory and begin
 * streaming q_w while the quantisation still runs, and reads q_a, s_tok only
 * after that kernel has completed.  q_w and s_ch must therefore not be written
 * by that quantisation (they are inputs of this call; nothing else runs in
 * between).  Workspace as for w8a8_scaled_mm (SQ_OP_W8A8). */
sq_status sq_w8a8_linear(const void* x_bf16, const float* inv_smooth, const int8_t* q_w,
                         const float* s_ch, void* y_bf16, int8_t* q_a, float* s_tok, int64_t M,
                         int64_t N, int64_t K, void* workspace, size_t ws_bytes, void* stream);

/* W8A8 with group-size-128 weight scales [P5]: s_blk fp32 [N, K/128], one
 * scale per (output row, 128-wide K block).  With P_kb[m,n] the exact int32
 * partial over block kb:  acc = 0; for kb ascending:
 * acc = fmaf(f32(P_kb), s_blk[n,kb], acc);  y = bf16_rne(acc * s_tok[m]).
 * Workspace as for w8a8_scaled_mm (SQ_OP_GS128; currently always 0). */
sq_status w8a8_gs128_mm(const int8_t* q_a, const float* s_tok, const int8_t* q_w,
                        const float* s_blk, void* y_bf16, int64_t M, int64_t N, int64_t K,
                        void* workspace, size_t ws_bytes, void* stream);

/* W8A16 weight-only GEMM [P1 "Recipe" item 2, P2]: x BF16 [M,K], q_w int8
 * [N,K], s_ch fp32 [N]; y = bf16_rne(s_ch[n] * sum_k x[m,k] * q_w[n,k]).
 * The int8 -> bf16 weight conversion is exact and the scale is applied in
 * the fp32 epilogue; products are exact and accumulate in fp32 (the order
 * of the fp32 sum is the kernel's).
 * M = 1 (K <= 30720) runs as a matrix-vector product on the CUDA cores in
 * exact integer arithmetic: the token becomes v = rint(x * 2^sh), |v| < 2^31
 * (sh from the exponent of max|x|; values more than 23 binades below the
 * largest are rounded to the nearest 2^-sh), the dot products with the codes
 * are exact (dp4a over the four bytes of v, combined in int64), and
 * y = bf16_rne(fp64(sum) * s_ch * 2^-sh).  A token holding inf or NaN has
 * no such image: every output of the call is then NaN.  Other small M
 * convert the weights on load into the tensor cores.
 * Workspace (SQ_OP_W8A16) holds split-K partials for small M (unused at
 * M = 1) and the converted BF16 weights for large M; the zero-fill rule of
 * w8a8_scaled_mm applies. */
sq_status w8a16_mm(const void* x_bf16, const int8_t* q_w, const float* s_ch, void* y_bf16,
                   int64_t M, int64_t N, int64_t K, void* workspace, size_t ws_bytes,
                   void* stream);

/* W8A8 GEMM that allocates nothing and takes no workspace.  The quantisation
 * pages have no counterpart: this exists for callers that cannot call
 * cudaMalloc, such as a plugin whose host framework owns all device memory and
 * passes only inputs and outputs, or a latency-critical thread on which
 * cudaMalloc would synchronise the device.  Same arguments, arithmetic and
 * results as w8a8_scaled_mm without the workspace.  For M <= 32 the split-K
 * partial sums live in a 5 MiB array in the library's static device memory
 * (held on every GPU that loads the library until the process exits); the
 * call returns SQ_ERR_WORKSPACE if these sizes would need more than that (not
 * the case on a 148-SM B200) and SQ_ERR_SHAPE if N > 2,097,152.  The first
 * call on a device looks up the array's device address (a synchronous runtime
 * call), so make it before any stream capture.  Every call shares the one
 * array and clears its counters first: calls that may overlap on the GPU (other
 * streams, other threads) race and must not be issued. */
sq_status w8a8_scaled_mm_noalloc(const int8_t* q_a, const float* s_tok, const int8_t* q_w,
                                 const float* s_ch, void* y_bf16, int64_t M, int64_t N,
                                 int64_t K, void* stream);

/* Next rows of the layer ----------------------------------------------- */

/* Norm weight with the SmoothQuant factor folded in [P1 "Recipe" item 1:
 * zero-centred norms absorb 1/s; P3 "Recipe" item 1]: gamma fp32 [K],
 * gamma[k] = f32(g_k * inv_smooth[k]) with g_k = 1 + f32(w_norm[k]) when
 * zero_centered != 0, else f32(w_norm[k]); inv_smooth may be NULL (= 1).
 * w_norm_bf16: BF16 [K]. */
sq_status sq_fold_norm_weight(const void* w_norm_bf16, int zero_centered,
                              const float* inv_smooth, float* gamma, int64_t K, void* stream);

/* Fused RMSNorm + SmoothQuant fold + dynamic INT8 quantisation [P1 "Recipe"
 * items 1-2, P5 "Serving": RMSNorm with per-group INT8 quantised output].
 * Per row m of h (BF16 [M,K]): ss = sum_k f32(h)^2 rounded once to fp32
 * (accumulated in fp64); r = 1 / sqrt(ss / K + eps) (IEEE fp32 division,
 * addition and square root); x'_k = (f32(h_k) * r) * gamma[k] (two fp32
 * roundings; gamma from sq_fold_norm_weight); then the quantisation of
 * sq_quant_per_token over the row (group == 0 or K: scales fp32 [M]) or over
 * each 128-column block (group == 128: scales fp32 [M, K/128]).  inv_rms
 * (fp32 [M], may be NULL) receives r.  eps > 0; K <= 24576.  The fp64 sum
 * of squares rounds to the exact sum's fp32 value except when that sum lies
 * within about K * 2^-53 (relative) of a point halfway between two fp32
 * numbers. */
sq_status sq_rmsnorm_quant(const void* h_bf16, const float* gamma, float eps, int64_t group,
                           int8_t* q_i8, float* scales, float* inv_rms, int64_t M, int64_t K,
                           void* stream);

/* Per-group (1 x 128) dynamic INT8 activation quantisation with the 1/s fold
 * [P5 "Serving": per-group INT8 quant-out]: sq_quant_per_token's arithmetic on
 * every 128-wide block of every row; s_a fp32 [M, K/128]. */
sq_status sq_quant_per_group(const void* x_bf16, const float* inv_smooth, int8_t* q_i8,
                             float* s_a, int64_t M, int64_t K, void* stream);

/* Per-group activations x gs128 weights [P5 "Why group_size 128", "Serving"]:
 * with P_kb the exact int32 partial over K block kb, acc = 0; for kb
 * ascending: acc = fmaf(f32(P_kb), f32(s_a[m,kb] * s_blk[n,kb]), acc);
 * y = bf16_rne(acc).  q_a int8 [M,K], s_a fp32 [M, K/128], q_w int8 [N,K],
 * s_blk fp32 [N, K/128] (sq_quant_weight with group 128).  Workspace as
 * for w8a8_scaled_mm (SQ_OP_PG128; currently always 0). */
sq_status w8a8_pg128_mm(const int8_t* q_a, const float* s_a, const int8_t* q_w,
                        const float* s_blk, void* y_bf16, int64_t M, int64_t N, int64_t K,
                        void* workspace, size_t ws_bytes, void* stream);

/* Group-wise W8A16 [P2 "Why W8A16 on Ampere": weight-only kernels
 * reconstruct 16-bit weights; eight integer bits with group-wise scaling]:
 * w_hat[n,k] = bf16_rne(f32(q_w[n,k] * s_grp[n, k/128])) (codes and scales
 * from sq_quant_weight with group 128), y = bf16_rne(sum_k x[m,k] *
 * w_hat[n,k]) with exact products accumulated in fp32 (the order of the
 * fp32 sum is the kernel's).  Workspace as for w8a16_mm (SQ_OP_W8A16_GROUP). */
sq_status w8a16_group_mm(const void* x_bf16, const int8_t* q_w, const float* s_grp,
                         void* y_bf16, int64_t M, int64_t N, int64_t K, void* workspace,
                         size_t ws_bytes, void* stream);

/* FP8 (OCP E4M3: bias 7, largest finite 448) per-group activations [P3b]:
 * per 128-wide block of each row, v = f32(x) * inv_smooth[k] (inv_smooth may
 * be NULL), amax = max|v|, s_a = amax / 448, code = e4m3_rne_satfinite(v *
 * (448 / amax)) (fp32 product); an all-zero block gives s_a = 0 and zero
 * codes.  q_e4m3 [M,K] (E4M3 bit patterns), s_a fp32 [M, K/128]; K <= 24576. */
sq_status sq_quant_fp8_per_group(const void* x_bf16, const float* inv_smooth, uint8_t* q_e4m3,
                                 float* s_a, int64_t M, int64_t K, void* stream);

/* FP8 block-scaled weights [P3b]: one scale per [128, 128] block of the
 * folded weight f32(w[n,k]) * smooth[k] (smooth may be NULL), with the
 * arithmetic of sq_quant_fp8_per_group over the block's 16384 values.
 * N % 128 == 0; q_e4m3 [N,K], s_w fp32 [N/128, K/128]. */
sq_status sq_quant_fp8_block(const void* w_bf16, const float* smooth, uint8_t* q_e4m3,
                             float* s_w, int64_t N, int64_t K, void* stream);

/* FP8 block-scaled GEMM [P3b]: tcgen05 E4M3 x E4M3 products accumulated in
 * fp32 per 128-wide K block (P_kb; the accumulation order inside a block is
 * the tensor core's), then acc = fmaf(P_kb, f32(s_a[m,kb] * s_w[n/128,kb]),
 * acc) for kb ascending, y = bf16_rne(acc).  N % 128 == 0.  Workspace as for
 * w8a8_scaled_mm (SQ_OP_FP8BLK; currently always 0). */
sq_status fp8_block_mm(const uint8_t* q_a, const float* s_a, const uint8_t* q_w,
                       const float* s_w, void* y_bf16, int64_t M, int64_t N, int64_t K,
                       void* workspace, size_t ws_bytes, void* stream);

/* Bytes of workspace an operation needs for these sizes (0 = none). */
size_t sq_workspace_bytes(int op, int64_t M, int64_t N, int64_t K);

/* Raw int32 accumulators of the W8A8 mainloop (same kernels, no epilogue):
 * acc int32 [M,N] = q_a . q_w^T.  Workspace as for SQ_OP_W8A8_I32. */
sq_status w8a8_mm_i32(const int8_t* q_a, const int8_t* q_w, int32_t* acc, int64_t M,
                      int64_t N, int64_t K, void* workspace, size_t ws_bytes, void* stream);

/* Offline preparation -------------------------------------------------- */

/* SmoothQuant factors from calibration maxima [P1 "Recipe" item 1]:
 * s_j = clamp(sqrt(max_m |x[m,j]|) / sqrt(max_n |w[n,j]|), floor_, cap)
 * computed in fp64 (alpha = 1/2); a column with both maxima zero gets 1, one
 * with only max|w| zero gets cap.  s_out[j] = f32(s_j),
 * inv_s_out[j] = f32(1 / s_out[j]).  x BF16 [M,K], w BF16 [N,K]; M, N >= 1. */
sq_status sq_smooth_factors(const void* x_bf16, int64_t M, const void* w_bf16, int64_t N,
                            int64_t K, double cap, double floor_, float* s_out,
                            float* inv_s_out, void* stream);

/* Symmetric INT8 weight quantisation of the folded weight W'[n,k] =
 * f32(w[n,k]) * smooth[k] [P1, P3, P4, P5]; smooth may be NULL.  group == 0:
 * scales fp32 [N] (per output channel); group == 128: scales fp32 [N, K/128].
 * Scale = amax/127, codes as in sq_quant_per_token. */
sq_status sq_quant_weight(const void* w_bf16, const float* smooth, int8_t* q_w, float* scales,
                          int64_t N, int64_t K, int64_t group, void* stream);

/* Launch policy ---------------------------------------------------------- */

/* Overlap of consecutive kernels (programmatic dependent launch; the pages
 * have no counterpart: it is a launch policy of this library).  enable != 0:
 * from now on, for calls made from the calling host thread only (other
 * threads keep the default), w8a8_scaled_mm, w8a8_mm_i32, w8a8_gs128_mm,
 * w8a8_pg128_mm, fp8_block_mm, w8a16_mm and w8a16_group_mm (M <= 32) launch
 * their GEMM so that it may start while the
 * kernel before it on the stream is still running: it requests its WEIGHT
 * tiles (q_w) at once and reads everything else (activations, scales,
 * workspace, output) only after that kernel has completed.  Enable it only
 * if no kernel that directly precedes such a call on its stream writes that
 * call's q_w.  enable == 0 (the default): every launch waits for the
 * preceding work as usual.  sq_w8a8_linear always overlaps its GEMM with its
 * own quantisation kernel.  Always returns SQ_OK. */
sq_status sq_set_overlap(int enable);

/* The schedule one GEMM call would use on a device with `sms` streaming
 * multiprocessors, worked out on the host alone (no GPU needed; the pages
 * have no counterpart: it describes this library's kernels).  op: SQ_OP_*.
 * kernel: 0 = CTA pairs (256 x 256 output tiles), 1 = one CTA per tile,
 * 2 = swapped small-M tiles on stream-K ranges (partial tiles meet in the
 * workspace), 3 = swapped small-M tiles whose K parts meet inside a
 * thread-block cluster (a call falls back to 2 when the device cannot hold
 * every cluster at once or the parts do not fit in shared memory),
 * 4 = block-scaled CTA pairs (gs128: 128 tokens x 256 channels, FP8 blocks:
 * 256 tokens x 128 channels per pair tile), 5 = W8A16 with one token on the
 * CUDA cores (a matrix-vector product, tile_n = most rows one CTA owns).
 * tile_m x tile_n: tokens x output channels per tile.  grid: CTAs (for
 * kernel 0 an upper bound: the launch takes the active-cluster limit).
 * splits: K parts per tile when every CTA owns one part of one tile, 0 when
 * the stream-K ranges cross tiles, 1 for whole-K tiles.  workspace_bytes: as
 * sq_workspace_bytes.  Returns SQ_ERR_SHAPE for sms <= 0 or a bad shape or op,
 * SQ_ERR_NULL for out == NULL. */
typedef struct {
  int32_t kernel;
  int32_t grid;
  int32_t tile_m;
  int32_t tile_n;
  int32_t splits;
  uint64_t workspace_bytes;
} sq_plan_info;

sq_status sq_describe_plan(int op, int64_t M, int64_t N, int64_t K, int sms,
                           sq_plan_info* out);

/* Tensor-pipe issue-rate probe (the pages have no counterpart: it measures
 * the roofline denominator of this device).  Launches, asynchronously on
 * `stream`, one CTA pair per two SMs (all resident at once), each issuing
 * `iters` back-to-back tcgen05.mma cta_group::2 instructions (M = 256,
 * N = 256, 32 bytes of K) from shared memory: kind 0 = INT8 (kind::i8,
 * int32 accumulators), 1 = FP8 E4M3 (kind::f8f6f4, fp32), 2 = BF16
 * (kind::f16, fp32).  *ops_per_launch receives the launch's multiply-add
 * count x 2; time the launch with events on `stream` and divide.
 * 2 <= iters <= 2^24. */
sq_status sq_mma_peak(int kind, int iters, void* stream, double* ops_per_launch);

/* Self-test of the timeout path (the pages have no counterpart).  Launches on
 * `stream` one thread that waits, with a limit of limit_cycles SM clock
 * cycles (0 < limit_cycles <= 4e9), on a barrier that nothing arrives on.
 * The wait gives up exactly as a GEMM role's wait does: it raises the kernel's
 * abort flag and latches the device error word, so sq_check_device_error
 * then returns SQ_ERR_TIMEOUT.  gave_up (device int) receives 1 when the
 * wait gave up through its own limit.  Nothing else runs in that kernel. */
sq_status sq_selftest_wait_timeout(int64_t limit_cycles, int* gave_up, void* stream);

/* Diagnostics ------------------------------------------------------------ */

/* Synchronises the current device, then returns SQ_ERR_TIMEOUT if any kernel
 * of this library latched a timeout since the last reset (reset != 0 clears
 * the word), SQ_ERR_CUDA if the device reports an error, else SQ_OK. */
sq_status sq_check_device_error(int reset);

const char* sq_status_string(sq_status s);

#ifdef __cplusplus
}
#endif
#endif
