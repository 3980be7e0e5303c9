/*
 * fp8blk.h - C ABI of the blockwise-E4M3 FP8 linear-layer library for
 * NVIDIA B200 (sm_100a).
 *
 * What the library computes
 * -------------------------
 * The Puro-2B-Base model card (friendli.ai; repeated on the alphaneural.io
 * card), in the training-setup paragraph under the Phase 1 / Phase 2 setting
 * table, says the main Transformer linear-layer GEMMs run in blockwise E4M3
 * FP8 and that numerically sensitive operations, master weights and
 * optimizer state stay in BF16/FP32.  The tech report (part 7/7, section 5,
 * related work) ties this to the FP8 mixed-precision recipe of DeepSeek-V3.
 * The pages fix no block size or scale format; this library defines them:
 *
 *   - activations: groups of 1x128 consecutive elements along the GEMM's
 *     contraction dimension; weights: 128x128 blocks;
 *   - scale s = amax / 448 as an IEEE float32 division, stored as float32
 *     (the dequantization multiplier; an all-zero group stores 0);
 *   - code = E4M3FN(x / s): IEEE float32 division, then round-to-nearest-
 *     even onto the OCP E4M3FN grid, saturating at +-448, sign kept
 *     (a negative value that rounds to zero is 0x80); 0 for s == 0;
 *   - GEMM: for every 128-wide contraction slab the tensor cores form an
 *     FP32 partial sum of code products, which is multiplied by the two
 *     scales of that slab and added to an FP32 accumulator ("promotion" at
 *     every slab); the result is rounded to BF16 (round-to-nearest-even).
 *
 * Layout conventions (every array dense and row-major: element [i][j] of an
 * [R, C] array is at i*C + j):
 *   activation, row-wise groups : codes u8 [rows, cols],
 *                                 scales f32 [cols/128, rows]
 *   activation, along-token groups (groups of 128 consecutive rows in each
 *   column, output transposed so tokens are contiguous):
 *                                 codes u8 [cols, rows],
 *                                 scales f32 [rows/128, cols]
 *   weight [n, k]               : codes u8 [n, k], optional transposed
 *                                 codes u8 [k, n], scales f32 [n/128, k/128]
 *   bf16 tensors are passed as pointers to 16-bit bfloat16 storage.
 *
 * Ownership and streams: the caller allocates and frees every buffer (device
 * memory unless stated).  No entry point allocates, frees, synchronizes or
 * keeps a pointer after it returns; all work is enqueued on `stream` (a
 * cudaStream_t passed as void*; NULL means the legacy default stream) on the
 * current CUDA device.  Outputs must not overlap inputs.
 *
 * Errors: arguments are checked on the host before anything is enqueued; a
 * failed check returns its status and enqueues nothing.  FP8_ERR_CUDA
 * reports a failed launch (cudaGetLastError after the launch).  Faults that
 * happen later on the device surface at the caller's next synchronization,
 * as with any CUDA work.  Every barrier wait inside a kernel is bounded in
 * time; a wait that runs out makes the kernel record FP8_ERR_TIMEOUT in a
 * sticky per-device error word (read it with fp8_get_error) and return
 * without completing its output.  Before it returns, a kernel still waits
 * (at most max(limit, 100 ms) per wait) for the copies and tensor-core
 * operations it has already issued.  The GEMM's two CTAs then meet at one
 * closing cluster barrier, which has no time limit of its own: both reach it
 * because every wait before it is bounded.
 */
#ifndef FP8BLK_H
#define FP8BLK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8_OK = 0,
    FP8_ERR_NULL = 1,     /* a required pointer is NULL                          */
    FP8_ERR_SHAPE = 2,    /* a size is negative, too large, or not a multiple of
                             128 where one is required                           */
    FP8_ERR_ALIGN = 3,    /* a pointer is not 16-byte aligned                     */
    FP8_ERR_MODE = 4,     /* an unknown mode value                                */
    FP8_ERR_CUDA = 5,     /* a CUDA runtime call or kernel launch failed          */
    FP8_ERR_TIMEOUT = 6   /* a bounded wait inside a kernel ran out (sticky)      */
} fp8_status;

/* Modes of fp8_quantize_act_1x128 (bit flags). */
enum {
    FP8_ROWWISE = 1,      /* groups along each row                     */
    FP8_COLWISE = 2,      /* groups along each column, transposed out  */
    FP8_BOTH = 3          /* both, from one read of the input          */
};

/* Largest contraction length (K of fprop, N of dgrad) the fprop/dgrad GEMMs
 * accept: 256 slabs of 128. */
#define FP8_MAX_CONTRACTION_FPROP 32768

/*
 * GEMM workspace.  Every GEMM entry point takes an optional device
 * workspace (workspace, workspace_bytes; NULL and 0 to go without).  With
 * one of at least fp8_gemm_workspace_bytes() bytes, a GEMM whose last wave
 * of 256x256 output tiles would leave more than 5% of the GPU's CTA pairs
 * idle, whose contraction has at least 32 slabs of 128, and whose work is
 * at least fp8_set_gemm_split_min_work's threshold per pair, cuts the tiles
 * of its last two waves into equal ranges of slabs, one range per pair; the
 * pair holding a tile's first slab adds the FP32 partial sums the other
 * pairs leave in the workspace (in a fixed order, so results are
 * reproducible run to run) before its epilogue.  Without a workspace every
 * tile is computed whole by one pair.  Either way every output element
 * satisfies the same error bound.
 *
 * The workspace is owned by the caller, 16-byte aligned, and must hold
 * zeros before its first use (cudaMemset); every call that completes leaves
 * it zeroed again.  After a call that reported FP8_ERR_TIMEOUT it must be
 * zeroed before reuse.  Two launches that may run at the same time (on
 * different streams) need different workspaces.  The size depends on the
 * device (about 19 MB on a 148-SM B200).
 */
fp8_status fp8_gemm_workspace_bytes(size_t *bytes);

/*
 * Least work per CTA pair, in units of one 256x256 tile times one slab of
 * 128, for which a GEMM given a workspace uses the split schedule (default
 * FP8_GEMM_SPLIT_MIN_WORK_DEFAULT).  Handing the partial sums over costs a few microseconds per launch,
 * so on a B200 the split gains only on long GEMMs: with it the 8192-token
 * gate_up wgrad (332 units per pair) ran 4% faster and the o_proj wgrad (55
 * units per pair) 10% slower.  0 lets the split apply whenever the other two
 * conditions hold.  Negative values return FP8_ERR_SHAPE.  Host-side
 * setting, shared by all devices and threads; it takes effect for launches
 * made after the call.
 */
#define FP8_GEMM_SPLIT_MIN_WORK_DEFAULT 160
fp8_status fp8_set_gemm_split_min_work(int64_t units_per_pair);

/*
 * Activation quantizer, 1x128 groups (row-wise) and/or 128x1 groups along
 * tokens (column-wise).  Row-wise groups serve fprop (X) and dgrad (dY);
 * column-wise groups serve wgrad, which contracts over tokens.
 * Passage: Puro-2B-Base model card (friendli.ai), training-setup paragraph
 * ("blockwise E4M3" linear-layer GEMMs); group shape and scale as defined at
 * the top of this header.
 *
 *   x_bf16  [rows, cols] bf16, 16-byte aligned.
 *   rows    >= 0; a multiple of 128 when mode includes FP8_COLWISE.
 *   cols    >= 0, a multiple of 128.
 *   mode    FP8_ROWWISE, FP8_COLWISE or FP8_BOTH.
 *   q_row   [rows, cols] u8 codes; s_row [cols/128, rows] f32 scales
 *           (written when mode & FP8_ROWWISE; may be NULL otherwise).
 *   q_colT  [cols, rows] u8 codes; s_col [rows/128, cols] f32 scales
 *           (written when mode & FP8_COLWISE; may be NULL otherwise).
 * All pointers used are 16-byte aligned.  rows == 0 or cols == 0 is a no-op
 * (pointers may then be NULL).
 */
fp8_status fp8_quantize_act_1x128(const void *x_bf16, int64_t rows, int64_t cols,
                                  int mode, uint8_t *q_row, float *s_row,
                                  uint8_t *q_colT, float *s_col, void *stream);

/*
 * Fused SwiGLU producer: h = bf16(bf16(silu(g)) * u) of a gate_up
 * activation, quantized like fp8_quantize_act_1x128 quantizes a bf16 H,
 * without writing H to memory.  g = gate_up[r, j] and u = gate_up[r, ffn + j]
 * for j < ffn (the gate rows of the fused gate_up weight come first).  silu
 * is rounded once, correctly, to bfloat16, then the product; the codes and
 * scales equal those of fp8_quantize_act_1x128 on that H bit for bit.
 * Passage: Puro-2B-Base model card (friendli.ai): model property table
 * (Qwen3-1.7B configuration, gated SiLU feed-forward of size 6144) and
 * training-setup paragraph (blockwise E4M3 linear-layer GEMMs, other
 * activations in BF16).
 *
 *   gate_up_bf16 [rows, 2 * ffn] bf16, 16-byte aligned.
 *   rows >= 0 and ffn >= 0, multiples of 128.
 *   mode, q_row, s_row, q_colT, s_col: as fp8_quantize_act_1x128 with
 *   cols = ffn (H is [rows, ffn]).
 * rows == 0 or ffn == 0 is a no-op (pointers may then be NULL).
 */
fp8_status fp8_swiglu_quantize_1x128(const void *gate_up_bf16, int64_t rows, int64_t ffn,
                                     int mode, uint8_t *q_row, float *s_row,
                                     uint8_t *q_colT, float *s_col, void *stream);

/*
 * RMSNorm's row statistic: rstd[i] = 1 / sqrt(mean_k x[i, k]^2 + eps),
 * with the sum of squares in FP64 and one rounding to FP32 (the correctly
 * rounded value except within 2^-40 of a rounding midpoint, where it may be
 * the neighbouring float).  Passage: Puro-2B-Base model card (friendli.ai),
 * model property table (Qwen3-1.7B configuration, exported as
 * Qwen3ForCausalLM, whose blocks normalize their input with RMSNorm; the
 * Transformers default eps is 1e-6).
 *
 *   x_bf16 [rows, cols] bf16, 16-byte aligned; rows >= 0, cols >= 0 a
 *          multiple of 8.
 *   eps    >= 0, finite.
 *   rstd   [rows] f32, 16-byte aligned.
 * rows == 0 or cols == 0 is a no-op (pointers may then be NULL).
 */
fp8_status fp8_rmsnorm_rstd(const void *x_bf16, int64_t rows, int64_t cols, float eps,
                            float *rstd, void *stream);

/*
 * Fused RMSNorm producer: y = bf16(gamma * bf16(fp32(x * rstd))) per
 * element (each rounding to nearest even; the order of the Transformers
 * Qwen3 RMSNorm: normalize in FP32, round to BF16, scale by the weight),
 * quantized like fp8_quantize_act_1x128 quantizes a bf16 y, without writing
 * y to memory.  Given the same rstd, the codes and scales equal those of
 * quantizing the unfused y bit for bit.  Passage: Puro-2B-Base model card,
 * model property table (Qwen3-1.7B configuration) and training-setup
 * paragraph (blockwise E4M3 linear-layer GEMMs on BF16 activations).
 *
 *   x_bf16     [rows, cols] bf16, 16-byte aligned; rows, cols >= 0,
 *              multiples of 128.
 *   rstd       [rows] f32 (for example from fp8_rmsnorm_rstd), 16-byte
 *              aligned.
 *   gamma_bf16 [cols] bf16 norm weight, 16-byte aligned.
 *   mode, q_row, s_row, q_colT, s_col: as fp8_quantize_act_1x128.
 * rows == 0 or cols == 0 is a no-op (pointers may then be NULL).
 */
fp8_status fp8_rmsnorm_quantize_1x128(const void *x_bf16, int64_t rows, int64_t cols,
                                      const float *rstd, const void *gamma_bf16, int mode,
                                      uint8_t *q_row, float *s_row, uint8_t *q_colT,
                                      float *s_col, void *stream);

/*
 * Weight quantizer, 128x128 blocks.
 * Passage: Puro-2B-Base model card, training-setup paragraph (blockwise E4M3);
 * the 128x128 block follows the DeepSeek-V3 recipe the Puro-2B tech report
 * cites (part 7/7, section 5).
 *
 *   w_bf16  [n, k] bf16, 16-byte aligned; n, k >= 0, multiples of 128.
 *   wq      [n, k] u8 codes.
 *   sw      [n/128, k/128] f32 block scales.
 *   wqT     [k, n] u8 transposed codes (the same bytes: a 128x128 block's
 *           scale does not depend on orientation), for dgrad; may be NULL.
 * n == 0 or k == 0 is a no-op (pointers may then be NULL).
 */
fp8_status fp8_quantize_weight_128x128(const void *w_bf16, int64_t n, int64_t k,
                                       uint8_t *wq, float *sw, uint8_t *wqT,
                                       void *stream);

/*
 * fprop: Y[m, n] = sum_k X[m, k] W[n, k]   (Y = X W^T), BF16 out.
 * Passage: Puro-2B-Base model card, training-setup paragraph (the main
 * linear-layer GEMMs run in blockwise E4M3, other tensors in BF16); per-slab
 * FP32 promotion after the DeepSeek-V3 recipe (tech report part 7/7, sec. 5).
 *
 *   xq [M, K] u8, sx [K/128, M] f32   - row-wise quantized X
 *   wq [N, K] u8, sw [N/128, K/128] f32 - 128x128 quantized W
 *   y_bf16 [M, N]
 *   M >= 0, a multiple of 128; N > 0 and K > 0, multiples of 128;
 *   K <= FP8_MAX_CONTRACTION_FPROP.  M == 0 is a no-op (pointers may then
 *   be NULL).
 *   workspace, workspace_bytes: see "GEMM workspace" above.
 */
fp8_status fp8_block_gemm_fprop(const uint8_t *xq, const float *sx, const uint8_t *wq,
                                const float *sw, void *y_bf16, int64_t M, int64_t N,
                                int64_t K, void *workspace, size_t workspace_bytes,
                                void *stream);

/*
 * dgrad: dX[m, k] = sum_n dY[m, n] W[n, k]   (dX = dY W), BF16 out.
 * Passage: as fprop (model card, training-setup paragraph; tech report part
 * 7/7, section 5).  The weight operand is the transposed copy of the codes,
 * which the weight quantizer writes beside the row-major ones, so that the
 * contraction over n runs along contiguous bytes.
 *
 *   dyq [M, N] u8, sdy [N/128, M] f32 - row-wise quantized dY (groups run
 *                                        along n, the contraction)
 *   wqT [K, N] u8                      - transposed weight codes from
 *                                        fp8_quantize_weight_128x128
 *   sw  [N/128, K/128] f32             - the weight's block scales (the
 *                                        same array fprop uses)
 *   dx_bf16 [M, K]
 *   M >= 0, a multiple of 128; N > 0 and K > 0, multiples of 128;
 *   N <= FP8_MAX_CONTRACTION_FPROP.  M == 0 is a no-op (pointers may then
 *   be NULL).
 *   workspace, workspace_bytes: see "GEMM workspace" above.
 */
fp8_status fp8_block_gemm_dgrad(const uint8_t *dyq, const float *sdy, const uint8_t *wqT,
                                const float *sw, void *dx_bf16, int64_t M, int64_t N,
                                int64_t K, void *workspace, size_t workspace_bytes,
                                void *stream);

/*
 * wgrad: dW[n, k] = sum_m dY[m, n] X[m, k]   (dW = dY^T X), contracting over
 * the M tokens, BF16 out.
 * Passage: as fprop (model card, training-setup paragraph; tech report part
 * 7/7, section 5).  Both operands are grouped along the tokens, so the
 * promotion coefficient of a slab is the outer product of the two scale
 * vectors.
 *
 *   dyqT [N, M] u8, sdyT [M/128, N] f32 - column-wise (along-token) dY
 *   xqT  [K, M] u8, sxT  [M/128, K] f32 - column-wise (along-token) X
 *   dw_bf16 [N, K]
 *   M > 0, N > 0, K > 0, all multiples of 128.
 *   workspace, workspace_bytes: see "GEMM workspace" above.
 */
fp8_status fp8_block_gemm_wgrad(const uint8_t *dyqT, const float *sdyT, const uint8_t *xqT,
                                const float *sxT, void *dw_bf16, int64_t N, int64_t K,
                                int64_t M, void *workspace, size_t workspace_bytes,
                                void *stream);

/*
 * wgrad accumulated into an FP32 main gradient: dW_f32[n, k] += sum_m
 * dY[m, n] X[m, k], with the same operands, promotion and error bound as
 * fp8_block_gemm_wgrad.  Each output element receives one FP32 addition
 * (round-to-nearest-even) of this call's FP32 result to the value in memory,
 * so successive micro-batches accumulate in place without a BF16 rounding.
 * Passage: Puro-2B-Base model card, training-setup paragraph (master weights
 * and optimizer state stay in FP32); the accumulation over the micro-batches
 * of one optimizer step follows from the setting table (global batch 1536,
 * micro-batch 2).
 *
 *   dyqT, sdyT, xqT, sxT, N, K, M, workspace, workspace_bytes - as
 *          fp8_block_gemm_wgrad
 *   dw_f32 [N, K] f32, read and written (16-byte aligned); must not overlap
 *          the inputs.  Calls on the same dw_f32 must be ordered (one stream).
 *          A sum below float32's normal range may be flushed to zero.
 */
fp8_status fp8_block_gemm_wgrad_accum_f32(const uint8_t *dyqT, const float *sdyT,
                                          const uint8_t *xqT, const float *sxT,
                                          float *dw_f32, int64_t N, int64_t K, int64_t M,
                                          void *workspace, size_t workspace_bytes,
                                          void *stream);

/*
 * wgrad fused with the data-parallel reduce-scatter of the weight gradient,
 * into FP32 main gradients: dW = dY^T X of this rank's tokens is added, as
 * fp8_block_gemm_wgrad_accum_f32 adds it, straight into the shard of the
 * rank that owns each row: rows [q N / nranks, (q + 1) N / nranks) of dW go
 * to dw_shards[q], a row-major [N / nranks, K] FP32 array.  Shards of other
 * GPUs are reached through peer mappings (CUDA IPC or peer access) with
 * vector reductions over NVLink, issued tile by tile as each 256 x 256 tile
 * of dW completes, so the transfer overlaps the GEMM.  When every rank of a
 * data-parallel group has made this call on its own tokens, and the group
 * has synchronized, shard q holds its previous contents plus the sum over
 * ranks: the reduce-scatter.  Additions from different ranks meet in
 * arbitrary order (each is one FP32 rounding).  Passage: Puro-2B-Base model
 * card (friendli.ai), Phase 1 / Phase 2 setting table (data parallelism 12
 * and 24) and training-setup paragraph (FP32 master state).
 *
 *   dyqT, sdyT, xqT, sxT, N, K, M, workspace, workspace_bytes - as
 *            fp8_block_gemm_wgrad (M = this rank's tokens)
 *   dw_shards  host array of nranks device pointers (this GPU's memory or
 *            a peer's, mapped into this process), each 16-byte aligned
 *   nranks   1 .. 8, dividing N
 * The shards must not overlap the inputs; calls that add into the same
 * shard on one GPU must be ordered (one stream), while calls of different
 * ranks may run at the same time (the reductions are atomic).
 */
fp8_status fp8_block_gemm_wgrad_reduce_scatter_f32(const uint8_t *dyqT, const float *sdyT,
                                                  const uint8_t *xqT, const float *sxT,
                                                  float *const *dw_shards, int nranks,
                                                  int64_t N, int64_t K, int64_t M,
                                                  void *workspace, size_t workspace_bytes,
                                                  void *stream);

/*
 * wgrad for callers that cannot allocate device memory: the same GEMM as
 * fp8_block_gemm_wgrad with the split schedule, whose workspace here is a
 * fixed array inside the library instead of a buffer the caller passes.
 * Some callers have no way to hand over a workspace: C code linked against
 * this library without a GPU memory manager of its own, or programs whose
 * framework allocator already holds (nearly) all device memory, or loops
 * that must not pay for cudaMalloc and cudaFree, which can synchronize the
 * device.  The pages have no counterpart to this entry point; it is a
 * packaging convenience of this library.
 *
 *   dyqT, sdyT, xqT, sxT, dw_bf16, N, K, M - as fp8_block_gemm_wgrad; the
 *   caller still owns and passes every input and output.
 *
 * Scratch: a file-scope device array of 24 MiB (enough for up to 94 CTA
 * pairs; a 148-SM B200 uses 74), which every GPU that loads the library
 * holds until the process exits.  A GPU that would need more returns
 * FP8_ERR_SHAPE (fp8_last_cuda_error says how much).  The first call on a
 * device looks up the array's device address and the GPU's CTA-pair count;
 * make that first call before any stream capture.  Every call clears the
 * array's flags with an asynchronous memset on `stream` and reuses the
 * array's previous contents otherwise, so calls that may run at the same
 * time on the GPU (different streams, or different host threads) race on
 * it: order them on one stream.  Nothing is allocated or freed.
 */
fp8_status fp8_block_gemm_wgrad_static_ws(const uint8_t *dyqT, const float *sdyT,
                                          const uint8_t *xqT, const float *sxT,
                                          void *dw_bf16, int64_t N, int64_t K, int64_t M,
                                          void *stream);

/* Sticky per-device error word: FP8_OK, or the first FP8_ERR_TIMEOUT a
 * kernel recorded on the current device since the last clear.  Reading it
 * synchronizes the device. */
fp8_status fp8_get_error(void);
fp8_status fp8_clear_error(void);

/* Time limit of every bounded wait inside the kernels launched after this
 * call, in nanoseconds (default 2e9; 0 restores the default).  Host-side
 * setting, shared by all devices and threads. */
fp8_status fp8_set_wait_timeout_ns(uint64_t ns);

/* Text for a status value (static storage). */
const char *fp8_status_string(fp8_status status);

/* Text of the last CUDA failure behind an FP8_ERR_CUDA returned to the
 * calling thread ("" if none): the failing call and CUDA's message.  The
 * storage is per thread and overwritten by the next failure. */
const char *fp8_last_cuda_error(void);

/* ----------------------------------------------------------- test support */

/* q[i] = E4M3FN(x[i] / scale) with the device rounding path the quantizers
 * use (IEEE float32 division, then round-to-nearest-even with saturation),
 * or 0 when scale == 0.  x: n f32 values; q: n bytes; n >= 0. */
fp8_status fp8_cast_e4m3_scaled(const float *x, float scale, uint8_t *q, int64_t n,
                                void *stream);

/* Exhaustive check of the quantizers' division path: for every positive
 * finite bf16 amax and every bf16 x with |x| <= amax, compares the E4M3
 * code (and the float32 quotient bits) the quantizers compute for x / s,
 * s = amax / 448, with those of the IEEE division.  result: 5 device
 * uint64 the caller zeroes, 16-byte aligned.  result[0] += code mismatches,
 * result[1] = first code mismatch (amax bits << 16 | x bits), result[2] +=
 * quotient-bit mismatches with |x / s| >= 2^-12, result[3] = first such,
 * result[4] += quotient-bit mismatches with |x / s| < 2^-12 (a range whose
 * codes are all zero). */
fp8_status fp8_selftest_division(unsigned long long *result, void *stream);

/* Launches one block whose only wait is on a barrier that nothing completes,
 * so that the bounded wait runs out after the current time limit and
 * records FP8_ERR_TIMEOUT in the sticky error word.  For testing the timeout
 * path; nothing else is touched. */
fp8_status fp8_selftest_wait_timeout(void *stream);

/* out[b] = the bfloat16 bits of silu(g) as fp8_swiglu_quantize_1x128
 * computes it, for the bfloat16 g with bits b, every b in 0..65535 (for
 * checking it exhaustively).  out: 65536 device uint16, 16-byte aligned.
 * Non-finite g are outside the definition. */
fp8_status fp8_selftest_silu_bf16(uint16_t *out, void *stream);

/* The GEMMs' work schedule, computed on the host by the same code the
 * kernel runs, for checking without a GPU: for an output of M x N over a
 * contraction of K, with `pairs` CTA pairs and split != 0 meaning "with a
 * workspace", writes one row of 5 int32 per segment of work, pair by pair
 * in execution order: pair, tile, first slab, one past the last slab, and
 * (first << 16 | end) of the range of pairs whose partial sums the segment
 * adds before its epilogue (first == end when none).  max_segs rows fit in
 * segs; *nsegs receives the count.  FP8_ERR_SHAPE for bad sizes or too many
 * segments. */
fp8_status fp8_selftest_gemm_schedule(int64_t M, int64_t N, int64_t K, int pairs, int split,
                                      int32_t *segs, int64_t max_segs, int64_t *nsegs);

/* Arms the next launch of a kernel family so that the first operand
 * barrier of every CTA (pair) expects 16 bytes more than its copies bring:
 * that wait runs out after the current time limit, the kernel
 * records FP8_ERR_TIMEOUT, drains what it issued and returns without
 * completing its output.  which: 1 = the next GEMM launch, 2 = the next
 * 128x128 tile quantizer launch (column-wise, both layouts or weights),
 * 3 = both.  Host-side flag shared by all threads and devices; each armed
 * family is disarmed by its next launch.  For testing the time-out path of
 * the real kernels; FP8_ERR_MODE for any other value. */
fp8_status fp8_selftest_stall_next(int which);

#ifdef __cplusplus
}
#endif

#endif /* FP8BLK_H */
