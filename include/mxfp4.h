/*
 * mxfp4.h -- C ABI of libmxfp4: MXFP4 quantization (optional randomized
 * Hadamard transform, round-to-nearest-even or stochastic rounding, 1D and 2D
 * blocks) and MXFP4 block-scaled GEMMs on NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page title and section:
 *   "MXFP4" (aiwiki.ai) -- "Format specification": E2M1 elements (values
 *       +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}), one E8M0 scale (2^(code-127), code
 *       0xFF = NaN) per block of 32, 136 bits per block.
 *     "Conversion rules": scale X = (largest power of two <= max|Vi|) / 4,
 *       elements Vi/X rounded to nearest-even and saturated to +-6; block dot
 *       products C = X(A) X(B) sum Pi(A) Pi(B) summed over blocks, FP32 result.
 *     "Clipping in the reference algorithm": shared exponent
 *       floor(log2 amax) - 2.
 *     "Training with MXFP4": stochastic rounding, random Hadamard transform,
 *       Hadamard size 32 for MXFP4.
 *     "Use in models / gpt-oss": blocks along the last dimension, two FP4
 *       values per byte, scales stored apart from the values.
 *   "Training an MoE LLM in MXFP4: How We Closed the Gap to BF16"
 *       (thesingularityreport.com), abstract: hybrid 1D/2D block quantization,
 *       randomized Hadamard transforms and stochastic rounding (the ALTO
 *       recipe on GPT-OSS-20B).
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates no device memory and keeps no pointer after returning.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Nothing synchronizes the host except mxfp4_get_error().
 *   - Arguments are validated before anything is launched; a failed check
 *     returns an error code and launches nothing.  Launch failures return
 *     MXFP4_ERR_CUDA.  Nothing crosses the ABI as an exception.
 *   - Leading dimensions: ld_x / ld_out in elements, ld_codes / ld_scales /
 *     lda / ldb in bytes, ldc in elements (ld_c_codes / ld_c_scales of the
 *     MXFP4-output GEMM in bytes).
 *   - Element codes: byte j of a 32-value block holds element 2j in bits 3:0
 *     and element 2j+1 in bits 7:4; bit 3 of a code is the sign.
 */
#ifndef MXFP4_H
#define MXFP4_H

#include <stdint.h>

#if defined(__GNUC__)
#define MXFP4_API __attribute__((visibility("default")))
#else
#define MXFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define MXFP4_OK 0
#define MXFP4_ERR_INVALID_ARG 1   /* null pointer, bad enum, shape outside the format */
#define MXFP4_ERR_ALIGNMENT 2     /* pointer or leading dimension not 16-byte aligned */
#define MXFP4_ERR_UNSUPPORTED 3   /* valid MXFP4 shape the library has no kernel for */
#define MXFP4_ERR_CUDA 4          /* a CUDA runtime/driver call failed */
#define MXFP4_ERR_TIMEOUT 5       /* a bounded device-side wait ran out (see mxfp4_get_error) */

/* Block layouts. */
#define MXFP4_LAYOUT_1D_ROW 0   /* 32 consecutive elements of a row */
#define MXFP4_LAYOUT_1D_COL 1   /* 32 consecutive elements of a column; stored transposed */
#define MXFP4_LAYOUT_2D 2       /* 32 x 32 tiles */

/* Element rounding (bits 3:0 of the `rounding` argument). */
#define MXFP4_ROUND_RNE 0
#define MXFP4_ROUND_SR 1
/* Scale rule (bits 5:4 of the `rounding` argument, OR-ed with the rounding).
 * "MXFP4" (aiwiki.ai), "Clipping in the reference algorithm" and the
 * "Training with MXFP4" table:
 *   FLOOR       the reference rule, code = floor(log2 amax) - 2 + 127;
 *   ROUNDUP     the decode scale amax / 6 rounded up to a power of two: the
 *               smallest e with 6 * 2^e >= amax, so no element saturates;
 *   PRESCALE_34 the FLOOR exponent (from the unscaled amax), and each element
 *               multiplied by 3/4 in fp32 before the division by the scale, so
 *               none reaches the clipping range.  The codes then hold 3/4 of
 *               the values: dequantize returns those, and a GEMM of two such
 *               operands returns 9/16 of the product; the caller undoes it. */
#define MXFP4_SCALE_FLOOR 0x00
#define MXFP4_SCALE_ROUNDUP 0x10
#define MXFP4_SCALE_PRESCALE_34 0x20

/* Scale storage. */
#define MXFP4_SCALES_ROWMAJOR 0 /* canonical: one byte per block, row-major */
#define MXFP4_SCALES_MMA 1      /* GEMM-ready, see mxfp4_mma_scale_offset */

/* Dequantize output type. */
#define MXFP4_OUT_BF16 0
#define MXFP4_OUT_F32 1

/* Human-readable name of a status code (static string, never NULL). */
MXFP4_API const char *mxfp4_status_string(int status);

/* ABI version (major * 100 + minor).  1.01 added mxfp4_gemm_bf16 and
 * mxfp4_grouped_gemm_bf16; 1.02 mxfp4_gemm_mxfp4; 1.03
 * mxfp4_grouped_gemm_wgrad_bf16; 1.04 mxfp4_scales_to_mma; 1.05
 * mxfp4_quantize_dual_rows. */
MXFP4_API int mxfp4_version(void);

/*
 * GEMM-ready ("MMA") scale layout of an operand with `rows` rows and `k`
 * elements per row (k a multiple of 32): one byte per (row, 32-element
 * K-block), grouped in 512-byte atoms of 128 rows x 4 K-blocks.  The byte of
 * (row, kb) sits at
 *     ((row / 128) * ceil(k / 128) + kb / 4) * 512
 *       + (row % 32) * 16 + ((row % 128) / 32) * 4 + kb % 4,
 * which is the order in which the sm_100a block-scaled MMA reads scale
 * factors from tensor memory after a 32x128-bit copy.  Rows are padded to a
 * multiple of 128 and K-blocks to a multiple of 4; pad bytes are never read
 * into a stored GEMM output.
 */
MXFP4_API int64_t mxfp4_mma_scales_bytes(int64_t rows, int64_t k);
MXFP4_API int64_t mxfp4_mma_scale_offset(int64_t row, int64_t kb, int64_t k);

/*
 * mxfp4_scales_to_mma -- canonical row-major E8M0 scales to the GEMM-ready
 * layout above, on the device.  ("MXFP4" (aiwiki.ai), "Use in models /
 * gpt-oss": one scale byte per 32-element block, stored apart from the
 * codes.)  For a caller that holds canonical scales -- from mxfp4_quantize
 * with MXFP4_SCALES_ROWMAJOR, or from elsewhere -- and wants to call the
 * GEMMs, which read only the GEMM-ready layout.
 *
 * scales: DEVICE, row-major with row stride ld_scales bytes:
 *   two_d = 0: [rows, k/32], one scale per row and K-block (1D blocks);
 *   two_d = 1: [rows/32, k/32], one scale per 32x32 tile (2D blocks, as
 *              mxfp4_quantize writes for MXFP4_LAYOUT_2D); each tile's scale
 *              is repeated on its 32 rows in the output.
 * mma_scales: DEVICE, mxfp4_mma_scales_bytes(rows, k) bytes, 4-byte aligned,
 *   fully overwritten (pad rows and pad K-blocks zero).  The two buffers must
 *   not overlap.
 * Requirements: rows > 0; k > 0, k % 32 == 0; rows % 32 == 0 when two_d;
 * ld_scales >= k / 32.  Reads 1 byte per block (1D) or per tile (2D), writes
 * the GEMM-ready bytes once: about 1/32 byte per element of the operand.
 */
MXFP4_API int mxfp4_scales_to_mma(const uint8_t *scales, int64_t ld_scales, int64_t rows, int64_t k, int two_d,
                                  uint8_t *mma_scales, void *stream);

/*
 * mxfp4_quantize -- bf16 tensor x[rows, cols] to MXFP4 codes and E8M0 scales.
 * ("Conversion rules"; RHT and SR from "Training with MXFP4"; 1D/2D blocks
 * from the ALTO abstract.)
 *
 * Per block: optional RHT y = c_d * H_d * diag(s) * x on each d-element
 * segment along the block axis (d = rht_size in {0 = off, 16, 32}; H_d the
 * Sylvester Hadamard matrix as an fp32 butterfly with stages h = 1, 2, .., d/2;
 * c_16 = 1/4, c_32 = fp32(1/sqrt(32)); s_j = -1 when bit j of word 0 of
 * Philox4x32-10(key = seed, counter = (0, 0, 0, 0x52485400)) is set); amax
 * over the block; scale code clamp(floor(log2 amax) - 2 + 127, 0, 254), or the
 * rule selected in bits 5:4 of `rounding` (MXFP4_SCALE_*) (0xFF
 * and all-zero element codes if the block holds a NaN or amax is Inf; code 0
 * if amax is 0); elements y * 2^-(code-127) rounded to E2M1 with saturation
 * at +-6, by nearest-even or, for MXFP4_ROUND_SR, up with probability
 * f = (|v| - lo)/(hi - lo) decided by r < f * 2^32, r = word (g mod 4) of
 * Philox4x32-10(key = seed, counter = (g/4, 0)) with g = linear index of the
 * element in the output view + elem_offset.  The sign bit is the sign of the
 * scaled value (a negative value rounding to zero is stored as -0).
 *
 * layout 1D_ROW: blocks along cols.  codes [rows, cols/2]; scales ROWMAJOR
 *                [rows, cols/32] or MMA for a (rows x cols) operand.
 * layout 1D_COL: blocks along rows, output in the transposed view: codes
 *                [cols, rows/2]; scales ROWMAJOR [cols, rows/32] or MMA for a
 *                (cols x rows) operand.  RHT runs along rows.
 * layout 2D:     32x32 tiles.  codes [rows, cols/2]; scales ROWMAJOR
 *                [rows/32, cols/32], or MMA for a (rows x cols) operand with
 *                each tile's scale repeated on its 32 rows.  RHT runs along
 *                cols.  codes_t (optional) [cols, rows/2] receives the
 *                transposed copy of the same codes; scales_t (optional)
 *                receives the scales of that transposed operand: ROWMAJOR
 *                [cols/32, rows/32] or MMA for a (cols x rows) operand.
 *
 * Requirements: rows, cols > 0; the block axis a multiple of 32 (both for 2D);
 * cols % 8 == 0; x, codes, codes_t 16-byte aligned; ld_x % 8 == 0;
 * ld_codes, ld_codes_t % 16 == 0; MMA scales 16-byte aligned;
 * elem_offset % 4 == 0.  ld_scales / ld_scales_t are ignored for MMA scales.
 * codes_t / scales_t must be NULL unless layout is 2D.
 */
MXFP4_API int mxfp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                   int layout, int rht_size, int rounding, uint64_t seed, uint64_t elem_offset,
                   uint8_t *codes, int64_t ld_codes,
                   uint8_t *scales, int64_t ld_scales, int scale_layout,
                   uint8_t *codes_t, int64_t ld_codes_t,
                   uint8_t *scales_t, int64_t ld_scales_t,
                   void *stream);

/*
 * mxfp4_quantize_dual -- both 1D layouts of one bf16 tensor x[rows, cols] from
 * a single read: row blocks (32 along cols, no RHT) into row_codes /
 * row_scales, exactly as mxfp4_quantize with MXFP4_LAYOUT_1D_ROW, and column
 * blocks (32 along rows, RHT of col_rht_size along rows) into col_codes /
 * col_scales, exactly as mxfp4_quantize with MXFP4_LAYOUT_1D_COL.  The ALTO
 * recipe ("Training an MoE LLM in MXFP4", abstract) quantizes activations and
 * gradients in both orientations: row blocks for the forward and data-gradient
 * GEMMs, blocks along tokens (with RHT) for the weight-gradient GEMM.  Both
 * outputs use `rounding` and `seed`; each output's SR stream index is the
 * element's index in its own output view plus row_elem_offset /
 * col_elem_offset.  Either output may be skipped by passing NULL codes.
 * Requirements: rows % 32 == 0, cols % 32 == 0, alignment as mxfp4_quantize.
 */
MXFP4_API int mxfp4_quantize_dual(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                                  int col_rht_size, int rounding, uint64_t seed,
                                  uint64_t row_elem_offset, uint64_t col_elem_offset,
                                  uint8_t *row_codes, int64_t ld_row_codes,
                                  uint8_t *row_scales, int64_t ld_row_scales,
                                  uint8_t *col_codes, int64_t ld_col_codes,
                                  uint8_t *col_scales, int64_t ld_col_scales,
                                  int scale_layout, void *stream);

/*
 * mxfp4_quantize_dual_rows -- mxfp4_quantize_dual of the row slice
 * [row0, row0 + rows) of a [total_rows, cols] tensor, producing exactly the
 * slice's part of the whole tensor's quantization.  For data-parallel
 * training that splits tokens across ranks (the ALTO recipe trains
 * GPT-OSS-20B, "Training an MoE LLM in MXFP4", abstract): each rank quantizes
 * its own tokens, and its codes and scales equal the whole batch's, stochastic
 * rounding included.
 *
 * x points at the slice's first row ([rows, cols], ld_x).  Row output: rows
 * [rows, cols/2] with SR indices row0 * cols + (r * cols + c), as
 * mxfp4_quantize_dual with row_elem_offset = row0 * cols.  Column output: the
 * whole tensor's column view is [cols, total_rows]; the slice is its column
 * range [row0, row0 + rows), written as [cols, rows/2] (ld_col_codes) with SR
 * indices c * total_rows + row0 + r -- which no single element offset can
 * express.  Column blocks of 32 tokens never straddle two slices because
 * row0 and total_rows are multiples of 32.  The RHT (col_rht_size) runs along
 * tokens within each block, as in mxfp4_quantize_dual.
 *
 * Requirements: as mxfp4_quantize_dual, plus 0 <= row0, row0 % 32 == 0,
 * total_rows % 32 == 0, row0 + rows <= total_rows.
 */
MXFP4_API int mxfp4_quantize_dual_rows(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int64_t row0,
                                       int64_t total_rows, int col_rht_size, int rounding, uint64_t seed,
                                       uint8_t *row_codes, int64_t ld_row_codes,
                                       uint8_t *row_scales, int64_t ld_row_scales,
                                       uint8_t *col_codes, int64_t ld_col_codes,
                                       uint8_t *col_scales, int64_t ld_col_scales,
                                       int scale_layout, void *stream);

/*
 * mxfp4_dequantize -- MXFP4 codes and scales back to a [rows, cols] tensor.
 * ("Format specification": value = E2M1(code) * 2^(scale - 127), the whole
 * block NaN for scale 0xFF.)  If rht_size != 0 the inverse transform
 * x = diag(s) * H_d * (c_d * y) (same butterfly order, same signs for `seed`)
 * runs on each segment before the store.  `layout`, codes and scales are as
 * written by mxfp4_quantize for a tensor of shape [rows, cols] (for 1D_COL
 * the codes are the transposed view [cols, rows/2]; for 2D the ROWMAJOR
 * scales are the [rows/32, cols/32] tile scales).  out_dtype MXFP4_OUT_BF16
 * (round to nearest even; exact without RHT) or MXFP4_OUT_F32; out has row
 * stride ld_out elements and must be 16-byte aligned with ld_out % 8 == 0.
 */
MXFP4_API int mxfp4_dequantize(const uint8_t *codes, int64_t ld_codes,
                     const uint8_t *scales, int64_t ld_scales, int scale_layout,
                     int64_t rows, int64_t cols, int layout, int rht_size, uint64_t seed,
                     void *out, int64_t ld_out, int out_dtype, void *stream);

/*
 * mxfp4_gemm -- C[M, N] = A[M, K] * B[N, K]^T in FP32, both operands MXFP4
 * with 32-element blocks along K.  ("Conversion rules": the block dot product
 * X(A) X(B) sum Pi(A) Pi(B), blocks summed, FP32 result; internal order is
 * the implementation's: FP32 accumulation per 64-element K step.)
 *
 * a_codes [M, K/2] (row stride lda bytes), a_scales MMA layout for (M x K);
 * b_codes [N, K/2] (ldb), b_scales MMA layout for (N x K); c [M, N] FP32
 * (row stride ldc elements), fully overwritten.  A 2D-quantized weight is
 * used as B through its codes (fprop) or its transposed copy (dgrad) with the
 * matching MMA scales.
 *
 * Requirements: M, N >= 1; K >= 64 and K % 64 == 0; code pointers, scale
 * pointers and c 16-byte aligned; lda, ldb % 16 == 0; ldc % 4 == 0.
 * Device-side waits are bounded; a wait that runs out records
 * MXFP4_ERR_TIMEOUT for mxfp4_get_error() and the kernel returns.
 */
MXFP4_API int mxfp4_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales,
               const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales,
               int64_t M, int64_t N, int64_t K, float *c, int64_t ldc, void *stream);

/*
 * mxfp4_grouped_gemm -- per group (expert) g:
 *     C[rows of g] = A[rows of g] * B_g^T
 * for MoE layers whose routed rows are sorted by expert.  Group g owns rows
 * [group_offsets[g], group_offsets[g] + group_sizes[g]) of A and C; every
 * group_offsets[g] must be a multiple of 128 (the row tile) and
 * group_offsets[g] + group_sizes[g] <= group_offsets[g+1]; rows between a
 * group's end and the next group's start are padding: never read into a
 * stored output and never written.  group_offsets (num_groups + 1 entries)
 * and group_sizes (num_groups entries) are DEVICE int32 arrays, read by the
 * kernel, so routing needs no host synchronization; a misaligned offset is
 * reported through mxfp4_get_error() as MXFP4_ERR_INVALID_ARG and its group
 * is skipped.
 *
 * a_codes [a_rows, K/2] (lda), a_scales MMA layout for (a_rows x K);
 * b_codes [num_groups, N, K/2] (ldb per row, groups contiguous), b_scales
 * num_groups consecutive MMA layouts for (N x K); c [a_rows, N] FP32 (ldc).
 * Requirements as for mxfp4_gemm; a_rows = group_offsets[num_groups].
 */
MXFP4_API int mxfp4_grouped_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, int64_t a_rows,
                       const int32_t *group_offsets, const int32_t *group_sizes, int num_groups,
                       const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales,
                       int64_t N, int64_t K, float *c, int64_t ldc, void *stream);

/*
 * mxfp4_gemm_bf16, mxfp4_grouped_gemm_bf16 -- the same products as
 * mxfp4_gemm and mxfp4_grouped_gemm with a bf16 output: each FP32 accumulator
 * is rounded to the nearest bf16 (ties to even) in the epilogue, so C costs
 * 2 bytes per element of HBM writes instead of 4.  c holds bf16 bit patterns
 * [M or a_rows, N] (row stride ldc elements), fully overwritten (grouped:
 * padding rows untouched).  The FP32 value rounded is the one mxfp4_gemm
 * would store.
 *
 * Requirements and errors as for the FP32 forms, except ldc % 8 == 0 (16-byte
 * rows for the tensor-memory-access stores).  This output form is one of the
 * fused GEMM epilogues the recipe's next step calls for (the pages quantize
 * and multiply but fix no output precision beyond FP32 accumulation).
 */
MXFP4_API int mxfp4_gemm_bf16(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales,
                              const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales,
                              int64_t M, int64_t N, int64_t K, uint16_t *c, int64_t ldc, void *stream);
MXFP4_API int mxfp4_grouped_gemm_bf16(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, int64_t a_rows,
                                      const int32_t *group_offsets, const int32_t *group_sizes, int num_groups,
                                      const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales,
                                      int64_t N, int64_t K, uint16_t *c, int64_t ldc, void *stream);

/*
 * mxfp4_gemm_mxfp4 -- the product of mxfp4_gemm requantized to MXFP4 in the
 * epilogue, for a next layer that takes C as a quantized operand: each run of
 * 32 FP32 results along a row of C (a 1D row block) gets the reference scale
 * rule and round-to-nearest-even E2M1 codes exactly as mxfp4_quantize would
 * give them for those FP32 values ("Conversion rules": amax, scale
 * X = 2^floor(log2 amax) / 4, saturating RNE; NaN or Inf in a block -> scale
 * 0xFF and zero codes).  The FP32 results themselves are never stored: C
 * costs 0.53 bytes per element of HBM writes instead of 4.
 *
 * c_codes [M, N/2] (row stride ld_c_codes bytes), c_scales row-major
 * [M, N/32] (ld_c_scales) or the GEMM-ready layout for (M x N)
 * (c_scale_layout MXFP4_SCALES_MMA, mxfp4_mma_scales_bytes(M, N) bytes), both
 * fully overwritten.  Operands and requirements as for mxfp4_gemm, plus
 * N % 32 == 0 and ld_c_codes % 16 == 0.  Because the FP32 accumulation order
 * is the implementation's, a block whose amax, or an element whose scaled
 * value, lies within the GEMM tolerance of a scale or rounding boundary may
 * take either neighbouring code.
 */
MXFP4_API int mxfp4_gemm_mxfp4(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales,
                               const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales,
                               int64_t M, int64_t N, int64_t K, uint8_t *c_codes, int64_t ld_c_codes,
                               uint8_t *c_scales, int64_t ld_c_scales, int c_scale_layout, void *stream);

/*
 * mxfp4_grouped_gemm_wgrad -- per group (expert) g:
 *     C_g[M, N] = sum over k in [group_offsets[g], group_offsets[g+1]) of
 *                 A[:, k] B[:, k]^T
 * the weight gradient of an MoE layer, dW_g = dY_g^T X_g, whose reduction
 * runs over the tokens routed to expert g.  ("Conversion rules": block dot
 * products summed in FP32; ALTO abstract: hybrid 1D/2D quantization, here the
 * 1D blocks along tokens of both operands.)  A and B are the 1D-column
 * quantizations of the expert-sorted routed tensors (dY [K, M] and X [K, N]),
 * so their blocks of 32 tokens never straddle two experts when every group
 * offset is a multiple of 128.
 *
 * a_codes [M, K/2] (lda bytes), a_scales MMA layout for (M x K); b_codes
 * [N, K/2] (ldb), b_scales MMA layout for (N x K); group_offsets: DEVICE int32
 * [num_groups + 1], multiples of 128, non-decreasing, group_offsets[num_groups]
 * <= K (token rows between a group's routed rows and the next offset are
 * padding and must be zero in A or B); c [num_groups * M, N] FP32 (ldc),
 * group g's output in rows [g * M, (g + 1) * M), fully overwritten (zero for
 * an empty group).  A bad offset is reported through mxfp4_get_error() as
 * MXFP4_ERR_INVALID_ARG and empties its group.
 *
 * Requirements: M, N >= 1; 1 <= num_groups <= 1024; K % 128 == 0; alignment
 * as for mxfp4_gemm.
 */
MXFP4_API int mxfp4_grouped_gemm_wgrad(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales,
                                       const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales,
                                       const int32_t *group_offsets, int num_groups, int64_t M, int64_t N,
                                       int64_t K, float *c, int64_t ldc, void *stream);

/*
 * mxfp4_grouped_gemm_wgrad_bf16 -- mxfp4_grouped_gemm_wgrad with a bf16
 * output: each FP32 accumulator rounded to the nearest bf16 (ties to even) in
 * the epilogue (an empty group's output is zero).  c holds bf16 bit patterns
 * [num_groups * M, N]; requirements as for mxfp4_grouped_gemm_wgrad except
 * ldc % 8 == 0.
 */
MXFP4_API int mxfp4_grouped_gemm_wgrad_bf16(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales,
                                            const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales,
                                            const int32_t *group_offsets, int num_groups, int64_t M, int64_t N,
                                            int64_t K, uint16_t *c, int64_t ldc, void *stream);

/*
 * NVFP4 ("MXFP4" (aiwiki.ai), "Comparison with NVFP4"): E2M1 elements in
 * blocks of 16, an FP8 E4M3 block scale, a second-level FP32 scale per
 * tensor; 4.5 bits per value.  The page gives the format, not the scale
 * rule; this library's rule: S = amax_tensor / 2688 (2688 = 6 * 448, so the
 * largest block scale is E4M3's maximum); block scale = E4M3 nearest-even of
 * amax_block / (6 S), saturating at 448; X = fp32(scale * S); elements
 * fp32(x / X) rounded to E2M1 (nearest-even, or MXFP4_ROUND_SR with the
 * Philox stream of mxfp4_quantize).  A block whose scale rounds to 0 stores
 * +-0; a NaN or Inf in the tensor gives every block the NaN scale 0x7F.
 *
 * mxfp4_nvfp4_quantize: computes the tensor amax into *tensor_amax (a DEVICE
 * float owned by the caller, overwritten; keep it for dequantize and the
 * GEMM), then quantizes.  layout 1D_ROW: blocks of 16 along cols, codes
 * [rows, cols/2], scales [rows, cols/16] bytes (ROWMAJOR) or the MMA layout
 * for a (rows x cols) NVFP4 operand (atoms of 4 blocks of 16); 1D_COL: blocks
 * along rows, transposed output (codes [cols, rows/2]).  No RHT.
 * Requirements: rows, cols multiples of 16; x, codes 16-byte aligned; ld_x %
 * 8 == 0; ld_codes % 16 == 0; elem_offset % 4 == 0; rounding RNE or SR.
 */
MXFP4_API int mxfp4_nvfp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int layout,
                                   int rounding, uint64_t seed, uint64_t elem_offset, float *tensor_amax,
                                   uint8_t *codes, int64_t ld_codes, uint8_t *scales, int64_t ld_scales,
                                   int scale_layout, void *stream);

/*
 * mxfp4_nvfp4_dequantize: out = fp32(fp32(code * scale) * S), S from the
 * DEVICE float *tensor_amax; out FP32 [rows, cols] (ld_out elements, 16-byte
 * aligned, ld_out % 4 == 0); layout and scale layout as for quantize.
 */
MXFP4_API int mxfp4_nvfp4_dequantize(const uint8_t *codes, int64_t ld_codes, const uint8_t *scales,
                                     int64_t ld_scales, int scale_layout, const float *tensor_amax, int64_t rows,
                                     int64_t cols, int layout, float *out, int64_t ld_out, void *stream);

/*
 * mxfp4_nvfp4_gemm: C[M, N] = S_a S_b * sum over 16-blocks of s_a s_b sum a b,
 * FP32 accumulation (tcgen05.mma kind::mxf4nvf4, UE4M3 scales per 16), the
 * second-level scales applied in the epilogue from the DEVICE floats a_amax,
 * b_amax written by mxfp4_nvfp4_quantize.  Scales in the MMA layout;
 * otherwise as mxfp4_gemm.
 */
MXFP4_API int mxfp4_nvfp4_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const float *a_amax,
                               const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales, const float *b_amax,
                               int64_t M, int64_t N, int64_t K, float *c, int64_t ldc, void *stream);

/*
 * mxfp4_get_error -- synchronize `stream`, then return and clear the first
 * error any kernel of this library recorded on the current device since the
 * last call (MXFP4_OK if none): MXFP4_ERR_TIMEOUT for a bounded wait that
 * ran out, MXFP4_ERR_INVALID_ARG for device-side argument checks.
 */
MXFP4_API int mxfp4_get_error(void *stream);

/*
 * mxfp4_set_wait_limit_ns -- limit, in nanoseconds of the GPU global timer,
 * of every device-side wait of later launches (default 2e9 = 2 s; 0 restores
 * the default).  Returns the previous limit.
 */
MXFP4_API uint64_t mxfp4_set_wait_limit_ns(uint64_t limit_ns);

/*
 * mxfp4_wait_probe -- test hook for the bounded-wait machinery: launches one
 * CTA that waits on a shared-memory barrier that `arrive` decides: if arrive
 * != 0 the kernel completes the barrier itself and the wait succeeds; if
 * arrive == 0 nothing ever completes it, the wait runs out after the wait
 * limit, records MXFP4_ERR_TIMEOUT and the kernel returns.  No copy, MMA or
 * tensor-memory allocation is in flight while it waits.
 */
MXFP4_API int mxfp4_wait_probe(int arrive, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MXFP4_H */
