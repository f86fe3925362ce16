/*
 * fp8q.h -- C ABI of the FP8 scaled-quantization library for NVIDIA B200
 * (sm_100a): amax -> scale -> saturating RNE cast to E4M3 / E5M2 -> FP8
 * scaled GEMM with fp32 accumulation and a bf16 epilogue, plus the
 * delayed-scaling amax-history update and the FP8 KV-cache quantize /
 * dequantize.
 *
 * Entry points, by step of the path
 *   amax and quantizers   fp8_amax, fp8_quantize_tensorwise (current or
 *                         delayed scale), fp8_quantize_rowwise (+ _pair for
 *                         both GEMM operands in one launch),
 *                         fp8_quantize_blockwise (1 x 128 / 128 x 128),
 *                         fp8_quantize_blockwise_e8m0 (power-of-two block
 *                         scales as the MMA's E8M0 image),
 *                         fp8_quantize_rowwise_transpose (per-row codes of
 *                         X^T for the bf16 weight-gradient recipe)
 *   GEMMs                 fp8_gemm_scaled (tensor / row / block scales),
 *                         fp8_gemm_block_e8m0, fp8_gemm_grouped (MoE groups),
 *                         fp8_gemm_bf16_wgrad; fp8_gemm_block_requant and
 *                         fp8_gemm_block_e8m0_requant quantize their own
 *                         output 1 x 128 for the next GEMM in the epilogue;
 *                         fp8_gemm_workspace_size / fp8_gemm_scaled_noalloc
 *                         for the split-K scratch
 *   delayed scaling       fp8_amax_history_update
 *   KV cache              fp8_kv_quant / fp8_kv_dequant (per (b, h) slice),
 *                         fp8_paged_kv_write / fp8_paged_kv_gather (pages)
 *   health and errors     fp8_scale_stats, fp8_device_error,
 *                         fp8_status_string
 *
 * Sources (web pages on FP8 scaled quantization):
 *   [DeepL]  "DeepL押注FP8：大模型训练与推理统一精度实战解析"
 *   [H100]   "H100 FP8加速实测：新一代计算架构的飞跃"
 *   [Soup]   "FP8训练与QAT量化感知训练：如何在Hopper GPU上用Soup把大模型微调提速2倍"
 *   Format bit semantics not fixed by the pages follow the OCP 8-bit
 *   floating point specification (E4M3: max 448, no Inf; E5M2: max 57344).
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is DEVICE memory owned by the caller (allocate it
 *     with cudaMalloc, torch, ...).  The library allocates nothing on the
 *     device and never synchronises the host; its only device state is
 *     static module memory: the sticky error words behind fp8_device_error
 *     and the scratch array of fp8_gemm_scaled_noalloc.
 *   - bf16 tensors are raw 16-bit bfloat16 words; FP8 tensors are one byte per
 *     element (the format's code); scales are IEEE fp32.
 *   - "scale" s multiplies before the cast (q = cast(x * s)); "scale_inv"
 *     d = 1 / s is what the GEMM and the dequantizer multiply by.
 *   - Layouts are row-major.  Data pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued asynchronously; the return value covers argument validation
 *     and the launch only.  Data-dependent events (non-finite inputs,
 *     saturation) are reported through the optional device counters.
 *   - Errors: FP8_ERR_INVALID_ARG (null pointer, bad enum), FP8_ERR_SHAPE
 *     (negative or unsupported extents), FP8_ERR_ALIGNMENT (pointer or
 *     leading dimension not aligned as stated), FP8_ERR_UNSUPPORTED_DEVICE
 *     (the current device is not compute capability 10.0), FP8_ERR_CUDA (a
 *     CUDA runtime call failed; the CUDA error is left for the caller).
 *     Nothing is enqueued when a call returns an error.
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FP8Q_API __attribute__((visibility("default")))
#else
#define FP8Q_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8_OK = 0,
    FP8_ERR_INVALID_ARG = 1,
    FP8_ERR_SHAPE = 2,
    FP8_ERR_ALIGNMENT = 3,
    FP8_ERR_UNSUPPORTED_DEVICE = 4,
    FP8_ERR_CUDA = 5
} fp8_status;

/* [DeepL] §2.1: E4M3 (1-4-3 bits) for forward weights and activations, E5M2
 * (1-5-2 bits, range +-57344 per [H100]) for gradients. */
typedef enum { FP8_E4M3 = 0, FP8_E5M2 = 1 } fp8_format;

/* [DeepL] §2.3 scaling granularity; [Soup] "FP8 三种缩放配方怎么选". */
typedef enum { FP8_SCALE_TENSOR = 0, FP8_SCALE_ROW = 1, FP8_SCALE_BLOCK = 2 } fp8_scale_mode;

/* Human-readable name of a status code (static string). */
FP8Q_API const char *fp8_status_string(fp8_status s);

/*
 * amax = max |x| over the finite elements of a bf16 tensor ([DeepL] §4.2:
 * the maximum absolute value per tensor).  NaN and +-Inf are excluded and
 * counted.
 *   x_bf16  [n] bf16, 16-byte aligned;  n >= 0 (n == 0 gives amax 0).
 *   amax    [1] fp32, overwritten.
 *   counts  [2] uint32 or NULL: counts[0] += number of non-finite elements.
 */
FP8Q_API fp8_status fp8_amax(const void *x_bf16, int64_t n, float *amax, uint32_t *counts, void *stream);

/*
 * Per-tensor quantization ([DeepL] §2.3 per-tensor scaling; [Soup] tensorwise
 * recipe) of a [rows, cols] bf16 tensor.
 *   scale_in == NULL : current scaling.  amax_out receives amax(x) and
 *                      s = fmax / amax (amax == 0 gives 1; overflow clamps
 *                      to FLT_MAX).  amax_out is REQUIRED in this mode.
 *                      Up to 65536 elements (without transpose_out) the
 *                      amax and the cast run in one launch (one CTA holding
 *                      the tensor in registers); larger tensors take an amax
 *                      launch, then a cast launch.
 *   scale_in != NULL : delayed scaling ([DeepL] §2.3): s = *scale_in (from
 *                      the amax history); amax_out (may be NULL) receives this
 *                      tensor's amax for the next history update.
 *   q             [rows, cols] FP8, or [cols, rows] when transpose_out != 0
 *                 (the transposed copy feeds the GEMM's B operand when the
 *                 weight is needed as W^T, e.g. a data-gradient GEMM).
 *   scale_inv_out [1] fp32: d = 1 / s.
 *   counts        [2] uint32 or NULL: [0] += non-finite inputs,
 *                 [1] += elements with |x * s| > fmax (saturated).
 *   Cast: q = RNE(fp32(x) * s) with saturation to +-fmax; NaN stays NaN.
 *   Shapes: rows, cols >= 0.  transpose_out requires rows % 16 == 0 and
 *   cols % 16 == 0.
 */
FP8Q_API fp8_status fp8_quantize_tensorwise(const void *x_bf16, int64_t rows, int64_t cols, fp8_format fmt,
                                   const float *scale_in, uint8_t *q, int transpose_out,
                                   float *scale_inv_out, float *amax_out, uint32_t *counts,
                                   void *stream);

/*
 * Per-row quantization ([DeepL] §2.3 per-row scaling; [Soup] rowwise recipe
 * with e4m3 and power-of-two scales) of x [rows, cols] with leading
 * dimension ld (elements).  pow2 != 0: s_r = the largest power of two with
 * amax_r * s_r <= fmax; pow2 == 0: s_r = fmax / amax_r.
 *   q          [rows, cols] FP8, dense.
 *   scale_inv  [rows] fp32, d_r = 1 / s_r.
 *   counts     [2] uint32 or NULL: [0] += non-finite inputs (NaN, +-Inf),
 *              [1] += saturated elements (|fp32(x) * s| > fmax: +-Inf and
 *              values whose scaled magnitude rounds past fmax; NaN is not
 *              saturated) -- [DeepL] §5.1: overflow and NaN are the failures
 *              to detect.  Added to, never reset; 4-byte aligned.
 *   Shapes: cols % 16 == 0, ld % 8 == 0, ld >= cols.
 */
FP8Q_API fp8_status fp8_quantize_rowwise(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                fp8_format fmt, int pow2, uint8_t *q, float *scale_inv,
                                uint32_t *counts, void *stream);

/*
 * Both operands of a rowwise GEMM in one launch: fp8_quantize_rowwise of
 * a [rows_a, cols] (leading dimension lda) into qa / sa and of b [rows_b,
 * cols] (ldb) into qb / sb, with the same format and scale rule (the
 * forward GEMM's activations and weights share K and E4M3).  One launch
 * instead of two saves a launch gap and a ramp on short tensors.  Shapes,
 * layouts and errors as fp8_quantize_rowwise; either count may be 0.
 * counts (as fp8_quantize_rowwise) adds both tensors' counts.
 */
FP8Q_API fp8_status fp8_quantize_rowwise_pair(const void *a_bf16, int64_t rows_a, int64_t lda, uint8_t *qa,
                                     float *sa, const void *b_bf16, int64_t rows_b, int64_t ldb, uint8_t *qb,
                                     float *sb, int64_t cols, fp8_format fmt, int pow2, uint32_t *counts,
                                     void *stream);

/*
 * Per-block quantization ([DeepL] §2.3: the tensor is cut into small blocks
 * with one scale each) of x [rows, cols] (leading dimension ld).  Blocks are
 * block_rows x 128: block_rows = 1 for activations (1x128), 128 for weights
 * (128x128).  Edge blocks use their valid elements.  s = fmax / amax_block.
 *   q          [rows, cols] FP8, dense.
 *   scale_inv  block_rows == 1  : [ceil(cols/128), rows]  (row index fastest,
 *                                  the layout the GEMM reads per K block);
 *              block_rows == 128: [ceil(rows/128), ceil(cols/128)].
 *   counts     [2] uint32 or NULL: [0] += non-finite inputs (NaN, +-Inf),
 *              [1] += saturated elements (|fp32(x) * s| > fmax: +-Inf and
 *              values whose scaled magnitude rounds past fmax; NaN is not
 *              saturated) -- [DeepL] §5.1: overflow and NaN are the failures
 *              to detect.  Added to, never reset; 4-byte aligned.
 *   Shapes: cols % 16 == 0, ld % 8 == 0, ld >= cols.
 */
FP8Q_API fp8_status fp8_quantize_blockwise(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                  fp8_format fmt, int block_rows, uint8_t *q, float *scale_inv,
                                  uint32_t *counts, void *stream);

/*
 * Rowwise quantization of the transpose, for the backward GEMMs ([Soup]
 * section "FP8 三种缩放配方怎么选": the rowwise recipes scale each row of
 * every GEMM operand; the weight gradient dW = dY^T X contracts over tokens
 * and the data gradient dX = dY W over output channels, so their K-major
 * operands are dY^T, X^T and W^T).  x [rows, cols] bf16 (leading dimension
 * ld); one scale per column c of x: pow2 != 0 gives the largest power of two
 * with amax_c * s_c <= fmax, pow2 == 0 gives s_c = fmax / amax_c (amax over
 * the finite entries of the column; 0 gives 1).
 *   qT         [cols, rows] FP8, dense: qT[c][r] = sat_RNE(fp32(x[r][c]) * s_c).
 *   scale_inv  [cols] fp32, 1 / s_c.
 *   amax_out   [cols] fp32, the column amax (on the three-launch path also
 *              the kernels' reduction buffer; overwritten).
 *   counts     [2] uint32 or NULL: [0] += non-finite inputs (NaN, +-Inf),
 *              [1] += saturated elements (|fp32(x) * s| > fmax: +-Inf and
 *              values whose scaled magnitude rounds past fmax; NaN is not
 *              saturated) -- [DeepL] §5.1: overflow and NaN are the failures
 *              to detect.  Added to, never reset; 4-byte aligned.
 *   Shapes: rows % 16 == 0, cols % 16 == 0, ld % 8 == 0, ld >= cols,
 *   ceil(rows / 64) <= 65535.  One launch when rows <= 16384 (x read once: an
 *   8-CTA cluster per 64-column strip combines its partial column maxima
 *   through distributed shared memory); longer columns take three launches:
 *   a memset of amax_out, the column reduction, the transposing cast.
 */
FP8Q_API fp8_status fp8_quantize_rowwise_transpose(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                          fp8_format fmt, int pow2, uint8_t *qT, float *scale_inv,
                                          float *amax_out, uint32_t *counts, void *stream);

/*
 * Per-block quantization with power-of-two scales written as an E8M0 scale
 * image, the operand format of the hardware block-scaled MMA
 * (fp8_gemm_block_e8m0).  Blocks as in fp8_quantize_blockwise ([DeepL] §2.3
 * per-block scaling; power-of-two scales as in [Soup]'s rowwise recipe):
 * s = the largest power of two with amax_block * s <= fmax (2^-126 ..
 * 2^127; amax 0 gives 1), q = sat_RNE(fp32(x) * s).
 *   q         [rows, cols] FP8, dense.
 *   sf_image  ceil(cols/512) * ceil(rows/128) * 512 bytes, 16-byte aligned.
 *             The dequantization factor of row r in K block kb (128 wide) is
 *             2^(e - 127) with e = sf_image[((kb / 4) * ceil(rows/128) + r/128)
 *             * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + kb % 4]: one
 *             byte per row and K block, four K blocks per 32-bit word (the
 *             block-scaled MMA's scale-factor layout).  Rows past `rows` in
 *             the last 128-row group: e = 127 when block_rows == 1, the
 *             block's e when block_rows == 128.  Bytes of K blocks past the
 *             last one are not written.
 *   counts    as fp8_quantize_blockwise.
 *   Shapes and errors: as fp8_quantize_blockwise.
 */
FP8Q_API fp8_status fp8_quantize_blockwise_e8m0(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                       fp8_format fmt, int block_rows, uint8_t *q, uint8_t *sf_image,
                                       uint32_t *counts, void *stream);

/*
 * FP8 scaled GEMM ([H100]: the multiply-accumulate runs on FP8 operands on
 * the tensor cores; [Soup] tensorwise / rowwise scaled matmuls; per-block
 * scales per [DeepL] §2.3):
 *   D[m, n] = bf16( scales * sum_k A[m, k] * B[n, k] ), fp32 accumulation.
 *   A  [M, K] FP8 (format fa), K contiguous.   B [N, K] FP8 (format fb), K
 *   contiguous (an nn.Linear weight [out, in]).  fa and fb may differ
 *   (E5M2 gradient x E4M3 weight).
 *   mode TENSOR: a_scale_inv [1], b_scale_inv [1]:  D = da*db*acc.
 *   mode ROW   : a_scale_inv [M], b_scale_inv [N]:  D = da[m]*db[n]*acc.
 *   mode BLOCK : a_scale_inv [ceil(K/128), M] (1x128 blocks of A),
 *                b_scale_inv [ceil(N/128), ceil(K/128)] (128x128 blocks of B):
 *                D = sum_kb da[kb, m] * db[n/128, kb] * acc_kb  (each 128-wide
 *                K block accumulated on the tensor cores, then promoted into
 *                an fp32 register accumulator with its two scales).
 *   D  [M, N] bf16 with leading dimension ldd (elements).
 *   workspace / workspace_bytes: optional device scratch (NULL, 0 = none).
 *       With at least fp8_gemm_workspace_size() bytes, a long-K problem
 *       (at least 64 K blocks of 128) whose 256 x 256 tiles fill at most half
 *       of the GPU's CTA pairs, and that the cluster split below does not
 *       take, has each tile computed as two K halves on two CTA pairs, the
 *       first half handing its fp32 partial to the second through the
 *       workspace (TENSOR and ROW modes, M > 128); with several waves of
 *       tiles whose last wave is at most half full, that wave's tiles are
 *       split the same way (their first halves run first, their second
 *       halves last).  The
 *       workspace must be zero-filled when first allocated; every call
 *       leaves it as it found it (its hand-off flags cleared), so the call
 *       may also be captured in a CUDA graph and replayed.  Calls that share
 *       a workspace must not overlap on the device.  A workspace belongs to
 *       one device.
 *   Few-tile problems split K without a workspace: when the 128 x 256
 *   tiles fill at most a quarter of the SMs and K has at least 8 blocks
 *   (any M), or at most half of them (M <= 128, decode-like shapes), each
 *   tile is computed by a thread-block cluster of S = 2..8 CTAs, CTA q
 *   accumulating K blocks [q*nk/S, (q+1)*nk/S) (nk = ceil(K/128)), and the
 *   partial tiles are summed through distributed shared memory in rank
 *   order (all three modes).  S is the largest value whose clusters are all
 *   resident at once, with at least two K blocks per part.
 *   The result is deterministic: a fixed K order per tile and a fixed
 *   summation order for split tiles (second half + first half; cluster ranks
 *   in order), so repeated calls with the same shapes and workspace setting
 *   on the same device are bit-identical.
 *   Shapes: M, N, K >= 0; K % 16 == 0; N % 8 == 0; ldd % 8 == 0, ldd >= N.
 *   K == 0 writes zeros.  workspace 16-byte aligned.
 */
FP8Q_API fp8_status fp8_gemm_scaled(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb,
                           int64_t M, int64_t N, int64_t K, fp8_scale_mode mode,
                           const float *a_scale_inv, const float *b_scale_inv, void *D_bf16,
                           int64_t ldd, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Block-scaled GEMM whose output is requantized for the next GEMM ([DeepL]
 * §2.3: per-block scales on every GEMM operand; an MLP's second GEMM takes
 * the first one's output, H = bf16(up(X)), quantized with 1 x 128 blocks).
 *   A, fa, B, fb, M, N, K, a_scale_inv, b_scale_inv: as fp8_gemm_scaled
 *       with mode FP8_SCALE_BLOCK (fp32 scales, 1 x 128 blocks of A,
 *       128 x 128 blocks of B).
 *   D_bf16 [M, N] bf16, leading dimension ldd, device: the GEMM output
 *       (RNE); may be NULL when M > 128 and K > 0, otherwise required.
 *   fo:          format of the requantized output.
 *   q            [M, N] FP8 (fo), dense, device, 16-byte aligned:
 *                q = fp8_quantize_blockwise(D, block_rows = 1, fo) code for
 *                code, whether or not D is stored.
 *   q_scale_inv  [ceil(N / 128), M] fp32, device: 1 / s of each row's
 *                128-column block (the layout fp8_quantize_blockwise
 *                writes for block_rows = 1).
 *   counts       [2] uint32 or NULL: non-finite and saturated elements of
 *                the requantization, as fp8_quantize_blockwise counts them.
 *   M > 128 and K > 0: one launch -- the CTA-pair kernel's epilogue rounds
 *   each output to bf16 and quantizes its 128-column blocks in registers
 *   (one thread holds one row of one block).  Otherwise two launches (the
 *   GEMM into D_bf16, then fp8_quantize_blockwise on it).
 *   Shapes: as fp8_gemm_scaled, and N % 16 == 0.  Errors as
 *   fp8_gemm_scaled; FP8_ERR_INVALID_ARG also for a NULL q or q_scale_inv,
 *   or a NULL D_bf16 where it is required.
 */
FP8Q_API fp8_status fp8_gemm_block_requant(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb,
                                  int64_t M, int64_t N, int64_t K, const float *a_scale_inv,
                                  const float *b_scale_inv, void *D_bf16, int64_t ldd, fp8_format fo,
                                  uint8_t *q, float *q_scale_inv, uint32_t *counts, void *stream);

/*
 * Weight-gradient GEMM kept in high precision ([Soup] section "FP8 三种缩放
 * 配方怎么选": the rowwise_with_gw_hp recipe keeps the weight gradient out of
 * FP8):
 *   dW[m, n] = (accumulate ? dW[m, n] : 0) + sum_t dY[t, m] * X[t, n],
 *   bf16 products accumulated in fp32 on the tensor cores, fp32 output.
 *   dY [T, M] bf16 (leading dimension ld_dy), X [T, N] bf16 (ld_x): the
 *   token-major tensors of the layer's backward pass, read as stored (no
 *   transpose pass).  dW [M, N] fp32, leading dimension ldd.
 *   Deterministic (one fixed token order per output).
 *   Shapes: M % 8 == 0, N % 8 == 0, ld_dy % 8 == 0, ld_x % 8 == 0,
 *   ldd % 4 == 0; T == 0 writes zeros (or leaves dW when accumulating).
 *   Pointers 16-byte aligned.
 */
FP8Q_API fp8_status fp8_gemm_bf16_wgrad(const void *dY_bf16, const void *X_bf16, int64_t T, int64_t M,
                               int64_t N, int64_t ld_dy, int64_t ld_x, float *dW, int64_t ldd,
                               int accumulate, void *stream);

/*
 * FP8 GEMM with power-of-two block scales applied by the tensor core
 * (tcgen05.mma.kind::mxf8f6f4.block_scale; [DeepL] §2.3 per-block scales):
 *   D[m, n] = bf16( sum_kb 2^(ea[m,kb] - 127) * 2^(eb[n,kb] - 127)
 *                   * sum_{k in kb} A[m, k] * B[n, k] ),  fp32 accumulation,
 *   exactly the BLOCK mode of fp8_gemm_scaled when its scales are powers of
 *   two, without the per-block promotion in the epilogue.
 *   A [M, K], B [N, K] FP8, K contiguous (formats fa, fb).
 *   a_sf, b_sf: E8M0 scale images of A and B in the layout
 *   fp8_quantize_blockwise_e8m0 writes (an exponent per row and 128-wide K
 *   block), 16-byte aligned, device.
 *   D [M, N] bf16, leading dimension ldd.  Deterministic (one fixed K order).
 *   Shapes: K % 16 == 0, N % 8 == 0, ldd % 8 == 0, ldd >= N; K == 0 writes
 *   zeros.  Errors as fp8_gemm_scaled.
 */
FP8Q_API fp8_status fp8_gemm_block_e8m0(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb,
                               int64_t M, int64_t N, int64_t K, const uint8_t *a_sf, const uint8_t *b_sf,
                               void *D_bf16, int64_t ldd, void *stream);

/*
 * fp8_gemm_block_e8m0 whose output is requantized for the next GEMM with
 * 1 x 128 blocks and power-of-two scales ([DeepL] §2.3 per-block scales;
 * [Soup]'s power-of-two scales): q and q_sf equal
 * fp8_quantize_blockwise_e8m0(D, block_rows = 1, fo) on D = bf16(GEMM),
 * code for code and byte for byte (rows past M in the last 128-row group:
 * e = 127; bytes of K blocks past the last one are not written).
 *   A, fa, B, fb, M, N, K, a_sf, b_sf: as fp8_gemm_block_e8m0.
 *   D_bf16 [M, N] bf16 (leading dimension ldd) or NULL: the GEMM output.
 *   q [M, N] FP8 (fo), dense, 16-byte aligned; q_sf the E8M0 image of q
 *   (fp8_quantize_blockwise_e8m0's layout and size for M x N), 16-byte
 *   aligned; counts [2] or NULL as the quantizers count.
 *   One launch: the epilogue rounds each output to bf16 and quantizes its
 *   row's 128-column block in registers.  K == 0: D = 0, codes 0, e = 127.
 *   Shapes: as fp8_gemm_block_e8m0, and N % 16 == 0.  Errors as
 *   fp8_gemm_block_e8m0; FP8_ERR_INVALID_ARG for a NULL q or q_sf.
 */
FP8Q_API fp8_status fp8_gemm_block_e8m0_requant(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb,
                                       int64_t M, int64_t N, int64_t K, const uint8_t *a_sf,
                                       const uint8_t *b_sf, void *D_bf16, int64_t ldd, fp8_format fo,
                                       uint8_t *q, uint8_t *q_sf, uint32_t *counts, void *stream);

/*
 * Grouped FP8 GEMM for mixture-of-experts layers ("DeepL押注FP8：…" §3.2: the
 * tokens routed to each expert form a group, and one grouped GEMM multiplies
 * every group by its own expert weight):
 *   for every group e:  D[r, :] = scales * A[r, :] x B_e^T  for the rows
 *   r in [group_offsets[e], group_offsets[e+1]).
 *   A  [total_M, K] FP8, the groups' rows stacked in order (K contiguous).
 *   B  [G, N, K] FP8, expert e's weight [N, K] at B + e*N*K.
 *   group_offsets  DEVICE int64 [G+1], group_offsets[0] = 0, nondecreasing,
 *                  group_offsets[G] = total_M (a group may be empty).
 *   mode TENSOR: a_scale_inv [G] (one per group's activations),
 *                b_scale_inv [G] (one per expert weight).
 *   mode ROW   : a_scale_inv [total_M], b_scale_inv [G*N].
 *   (BLOCK is not supported here: FP8_ERR_INVALID_ARG.)
 *   D  [total_M, N] bf16, leading dimension ldd.
 *   Same arithmetic, determinism and alignment rules as fp8_gemm_scaled;
 *   total_M < 2^30, G*N < 2^30.
 */
FP8Q_API fp8_status fp8_gemm_grouped(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb, int G,
                                     const int64_t *group_offsets, int64_t total_M, int64_t N, int64_t K,
                                     fp8_scale_mode mode, const float *a_scale_inv, const float *b_scale_inv,
                                     void *D_bf16, int64_t ldd, void *stream);

/*
 * Bytes of workspace fp8_gemm_scaled can use for this shape on the current
 * device (0: no pair split applies -- the shape fills whole waves, K is
 * short, the cluster split takes it, or the mode takes none).
 */
FP8Q_API fp8_status fp8_gemm_workspace_size(int64_t M, int64_t N, int64_t K, fp8_scale_mode mode,
                                            size_t *bytes);

/*
 * fp8_gemm_scaled for callers that cannot allocate device memory where they
 * run the GEMM (for example code inside a framework whose own caching
 * allocator owns every device byte, or latency-critical paths that cannot
 * afford cudaMalloc's implicit device synchronisation).  The source pages
 * have no counterpart to this entry point; it is a service of this library.
 *   Same arguments and result as fp8_gemm_scaled without the workspace: the
 *   split-K scratch comes from a 10 MiB array built into the library, which
 *   every GPU that loads the library holds until the process exits.  The
 *   caller still passes A, B, the scales and D.
 *   Returns FP8_ERR_SHAPE when the shape's split needs more scratch than the
 *   10 MiB (fp8_gemm_workspace_size() > 10 MiB); nothing is enqueued then.
 *   On a 148-SM B200 the largest split needs 9.25 MiB (37 tiles of two
 *   128 x 256 fp32 partials), so every shape runs there.
 *   The first call on a device that needs the scratch does a one-time
 *   set-up: it looks up the array's device address (the array starts
 *   zeroed when the library's module loads, and each call leaves its
 *   hand-off flags zeroed); make that first call before any stream capture.
 *   Allocates nothing: no cudaMalloc / cudaFree or allocating library call.
 *   All calls on a device share the one array and it keeps the last call's
 *   contents; calls that overlap on the GPU (other streams, other threads)
 *   race on it.
 */
FP8Q_API fp8_status fp8_gemm_scaled_noalloc(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb,
                                            int64_t M, int64_t N, int64_t K, fp8_scale_mode mode,
                                            const float *a_scale_inv, const float *b_scale_inv, void *D_bf16,
                                            int64_t ldd, void *stream);

/*
 * Delayed-scaling update ([DeepL] §2.3: the scale of a step is predicted
 * from the statistics of previous steps; a deviation above a threshold
 * forces recomputation).  In order:
 *   *saturated = (amax_cur * scale_t > fmax)   [the scale in use could not
 *                                               represent this step's amax]
 *   history[*pos] = amax_cur;  *pos = (*pos + 1) % len;
 *   *scale = fmax / max(history) (1 if the max is 0);  *scale_inv = 1 / *scale.
 *   history [len] fp32, pos [1] int32, amax_cur [1] fp32, scale / scale_inv
 *   [1] fp32 (scale is read as scale_t, then overwritten), saturated [1]
 *   uint32.  1 <= len <= 1024.  The state (history, pos, scale) is the whole
 *   checkpoint.
 */
FP8Q_API fp8_status fp8_amax_history_update(float *history, int32_t *pos, int len, const float *amax_cur,
                                   fp8_format fmt, float *scale, float *scale_inv,
                                   uint32_t *saturated, void *stream);

/*
 * FP8 KV-cache quantization ([DeepL] §3.1: K and V stored in FP8 halve the
 * cache).  kv [B, H, S, Dh] bf16; each (b, h) slice of S*Dh elements gets a
 * per-tensor scale s = fmax / amax(slice).
 *   q          [B, H, S, Dh] FP8.   scale_inv [B*H] fp32.
 *   counts     [2] uint32 or NULL: [0] += non-finite inputs, [1] += saturated
 *              elements (as fp8_quantize_rowwise); 4-byte aligned.
 *   Shapes: (S*Dh) % 16 == 0, B*H <= 65535.
 */
FP8Q_API fp8_status fp8_kv_quant(const void *kv_bf16, int64_t B, int64_t H, int64_t S, int64_t Dh,
                        fp8_format fmt, uint8_t *q, float *scale_inv, uint32_t *counts, void *stream);

/*
 * FP8 KV-cache dequantization when the cache is read ([DeepL] §3.1):
 *   out = bf16_RNE(fp32(q) * scale_inv[b*H + h]).
 *   q [B, H, S, Dh] FP8, scale_inv [B*H], out [B, H, S, Dh] bf16.
 *   Shapes: (S*Dh) % 16 == 0, B*H <= 65535.
 */
FP8Q_API fp8_status fp8_kv_dequant(const uint8_t *q, const float *scale_inv, int64_t B, int64_t H,
                          int64_t S, int64_t Dh, fp8_format fmt, void *out_bf16, void *stream);

/*
 * Paged FP8 KV cache, write side ("ms-swift全链路能力解析：训练、推理、评测、量化与
 * 部署一体化解决方案": the KV cache is cut into fixed-size blocks allocated on demand;
 * [DeepL] §3.1: K and V stored in FP8).  Each (token, head) row of Dh
 * elements is quantized with its own scale s = fmax / amax(row) (tokens
 * arrive a few at a time, so a per-sequence amax is not known yet).
 *   kv_bf16       [T, H, Dh] bf16, device, 16-byte aligned.
 *   slot_mapping  [T] int64, device: slot = block * block_size + offset of
 *                 each token; a slot outside [0, num_slots) marks padding and
 *                 writes nothing.  Slots must be distinct (otherwise which
 *                 token lands in a shared slot is unspecified).
 *   cache         [num_slots, H, Dh] FP8 (= [num_blocks, block_size, H, Dh]),
 *                 device, 16-byte aligned; only the mapped slots are written.
 *   scale_cache   [num_slots, H] fp32, device: 1/s of each written row.
 *   Shapes: Dh % 8 == 0, H * Dh <= 8192.
 *   Errors: FP8_ERR_SHAPE, FP8_ERR_INVALID_ARG (NULL pointer, format),
 *   FP8_ERR_ALIGNMENT.
 */
FP8Q_API fp8_status fp8_paged_kv_write(const void *kv_bf16, const int64_t *slot_mapping, int64_t T,
                              int64_t H, int64_t Dh, int64_t num_slots, fp8_format fmt, uint8_t *cache,
                              float *scale_cache, void *stream);

/*
 * Paged FP8 KV cache, read side: every sequence's tokens read back through
 * its block table, dequantized ([DeepL] §3.1):
 *   out[b][t][h][:] = bf16_RNE(fp32(q) * scale_cache[slot][h]),
 *   slot = block_table[b][t / block_size] * block_size + t % block_size.
 *   block_table [B, max_blocks] int32, seq_lens [B] int32, device.
 *   out         [B, S_out, H, Dh] bf16, device, 16-byte aligned; a position
 *               t >= seq_lens[b], past max_blocks * block_size, or whose
 *               block id is outside [0, num_blocks) is written as 0.
 *   Shapes: Dh % 8 == 0, H * Dh <= 8192, B <= 65535, block_size >= 1.
 *   Errors: as fp8_paged_kv_write.
 */
FP8Q_API fp8_status fp8_paged_kv_gather(const uint8_t *cache, const float *scale_cache,
                               const int32_t *block_table, const int32_t *seq_lens, int64_t B,
                               int64_t max_blocks, int64_t H, int64_t Dh, int64_t block_size,
                               int64_t num_blocks, int64_t S_out, fp8_format fmt, void *out_bf16,
                               void *stream);

/*
 * Health check of scale factors ([DeepL] §6.2: report the min / max / mean of
 * each layer's scales at intervals; a step change in a scale signals an
 * outlier or a drift of the data distribution).
 *   scales      [n] fp32, device.  Segment g covers
 *               scales[seg_offsets[g] .. seg_offsets[g+1]) (device int64
 *               [num_segments + 1], non-decreasing, clamped to [0, n] on the
 *               device); seg_offsets == NULL means one segment, the whole
 *               array (num_segments must then be 1).
 *   prev        [n] fp32, device, the previous snapshot of the same scales, or
 *               NULL (no step-change check).
 *   jump_ratio  >= 1: an entry is a step change when it and its previous value
 *               are both valid and either ratio (fp32 division) exceeds it.
 *   stats       [num_segments][3] fp32, device: {min, max, mean} over the
 *               valid entries (finite and > 0); mean = fp64 sum / count,
 *               rounded to fp32; all three 0 when a segment has none.
 *   counts      [num_segments][2] uint32, device: {step changes, invalid
 *               entries (NaN, +-Inf, <= 0)}.
 *   Deterministic: a fixed reduction order per segment.  n < 2^32.
 *   Errors: FP8_ERR_INVALID_ARG (NULL output, jump_ratio < 1 or not finite),
 *   FP8_ERR_SHAPE (segment count).
 */
FP8Q_API fp8_status fp8_scale_stats(const float *scales, const float *prev, int64_t n,
                           const int64_t *seg_offsets, int64_t num_segments, float jump_ratio,
                           float *stats, uint32_t *counts, void *stream);

/*
 * Device error word of the library on the current device: a bit is set when
 * a kernel gave up a bounded wait (a pipeline barrier that did not complete
 * within about one second) and returned early instead of hanging.  0 means
 * no such event.  Synchronises the current device.  clear != 0 resets it.
 */
FP8Q_API fp8_status fp8_device_error(uint32_t *host_out, int clear);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
