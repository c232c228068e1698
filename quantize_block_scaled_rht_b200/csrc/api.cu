// api.cu -- the extern "C" boundary of libmxfp4 (declared in include/mxfp4.h):
// argument validation, then one launch on the caller's stream.  No device
// memory is allocated here; errors come back as status codes.
#include <cstdint>

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace mxfp4 {
cudaError_t launch_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int layout, int rht,
                            int rounding, uint64_t seed, uint64_t elem_offset, uint8_t *codes, int64_t ld_codes,
                            uint8_t *scales, int64_t ld_scales, int scale_layout, uint8_t *codes_t,
                            int64_t ld_codes_t, uint8_t *scales_t, int64_t ld_scales_t, cudaStream_t s);
cudaError_t launch_quantize_dual(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int col_rht, int rounding,
                                 uint64_t seed, uint64_t row_offset, uint64_t col_offset, uint8_t *rcodes,
                                 int64_t ld_rcodes, uint8_t *rscales, int64_t ld_rscales, uint8_t *ccodes,
                                 int64_t ld_ccodes, uint8_t *cscales, int64_t ld_cscales, int scale_layout,
                                 int64_t col_sr_ld, cudaStream_t s);
cudaError_t launch_dequantize(const uint8_t *codes, int64_t ld_codes, const uint8_t *scales, int64_t ld_scales,
                              int scale_layout, int64_t rows, int64_t cols, int layout, int rht, uint64_t seed,
                              void *out, int64_t ld_out, int out_dtype, cudaStream_t s);
int launch_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes, int64_t ldb,
                const uint8_t *b_scales, int64_t M, int64_t N, int64_t K, float *c, int64_t ldc, cudaStream_t s);
int launch_grouped_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, int64_t a_rows,
                        const int32_t *offsets, const int32_t *sizes, int G, const uint8_t *b_codes, int64_t ldb,
                        const uint8_t *b_scales, int64_t N, int64_t K, float *c, int64_t ldc, cudaStream_t s);
int launch_grouped_wgrad(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes,
                         int64_t ldb, const uint8_t *b_scales, const int32_t *offsets, int G, int64_t M, int64_t N,
                         int64_t K, float *c, int64_t ldc, cudaStream_t s);
int launch_gemm_bf16(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes,
                     int64_t ldb, const uint8_t *b_scales, int64_t M, int64_t N, int64_t K, uint16_t *c, int64_t ldc,
                     cudaStream_t s);
int launch_gemm_mx(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes,
                   int64_t ldb, const uint8_t *b_scales, int64_t M, int64_t N, int64_t K, uint8_t *c_codes,
                   int64_t ld_c_codes, uint8_t *c_scales, int64_t ld_c_scales, int c_scale_mma, cudaStream_t s);
int launch_grouped_wgrad_bf16(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes,
                              int64_t ldb, const uint8_t *b_scales, const int32_t *offsets, int G, int64_t M,
                              int64_t N, int64_t K, uint16_t *c, int64_t ldc, cudaStream_t s);
int launch_grouped_gemm_bf16(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, int64_t a_rows,
                             const int32_t *offsets, const int32_t *sizes, int G, const uint8_t *b_codes,
                             int64_t ldb, const uint8_t *b_scales, int64_t N, int64_t K, uint16_t *c, int64_t ldc,
                             cudaStream_t s);
cudaError_t launch_nvfp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int layout, int rounding,
                                  uint64_t seed, uint64_t elem_offset, float *tensor_amax, uint8_t *codes,
                                  int64_t ld_codes, uint8_t *scales, int64_t ld_scales, int scale_layout,
                                  cudaStream_t s);
cudaError_t launch_nvfp4_dequantize(const uint8_t *codes, int64_t ld_codes, const uint8_t *scales, int64_t ld_scales,
                                    int scale_layout, const float *tensor_amax, int64_t rows, int64_t cols,
                                    int layout, float *out, int64_t ld_out, cudaStream_t s);
int launch_nvfp4_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const float *a_amax,
                      const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales, const float *b_amax, int64_t M,
                      int64_t N, int64_t K, float *c, int64_t ldc, cudaStream_t s);
cudaError_t launch_scales_to_mma(const uint8_t *src, int64_t ld_src, int64_t rows, int64_t k, int two_d,
                                 uint8_t *dst, cudaStream_t s);
int get_error(cudaStream_t s);
int launch_wait_probe(int arrive, cudaStream_t s);
uint64_t set_wait_limit(uint64_t ns);
}  // namespace mxfp4

namespace {
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An NVTX range around each entry point that enqueues work, so a profiler's
// timeline shows the library call that launched each kernel.  Without a tool
// attached NVTX calls return at once.
struct Range {
    explicit Range(const char *name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
    Range(const Range &) = delete;
    Range &operator=(const Range &) = delete;
};
}  // namespace

extern "C" {

const char *mxfp4_status_string(int status) {
    switch (status) {
        case MXFP4_OK: return "MXFP4_OK";
        case MXFP4_ERR_INVALID_ARG: return "MXFP4_ERR_INVALID_ARG";
        case MXFP4_ERR_ALIGNMENT: return "MXFP4_ERR_ALIGNMENT";
        case MXFP4_ERR_UNSUPPORTED: return "MXFP4_ERR_UNSUPPORTED";
        case MXFP4_ERR_CUDA: return "MXFP4_ERR_CUDA";
        case MXFP4_ERR_TIMEOUT: return "MXFP4_ERR_TIMEOUT";
        default: return "MXFP4_ERR_UNKNOWN";
    }
}

int mxfp4_version(void) { return 105; }

int64_t mxfp4_mma_scales_bytes(int64_t rows, int64_t k) {
    if (rows <= 0 || k <= 0) return 0;
    return ((rows + 127) / 128) * mxfp4::mma_katoms(k) * 512;
}

int64_t mxfp4_mma_scale_offset(int64_t row, int64_t kb, int64_t k) {
    return mxfp4::mma_scale_off(row, kb, mxfp4::mma_katoms(k));
}

// `rounding` = element rounding (bits 3:0) | scale rule (bits 5:4); no other bits.
static bool valid_rounding(int rounding) {
    const int rnd = rounding & 0x0F, rule = rounding & 0x30;
    if ((rounding & ~0x3F) != 0) return false;
    if (rnd != MXFP4_ROUND_RNE && rnd != MXFP4_ROUND_SR) return false;
    return rule == MXFP4_SCALE_FLOOR || rule == MXFP4_SCALE_ROUNDUP || rule == MXFP4_SCALE_PRESCALE_34;
}

int mxfp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int layout, int rht_size, int rounding,
                   uint64_t seed, uint64_t elem_offset, uint8_t *codes, int64_t ld_codes, uint8_t *scales,
                   int64_t ld_scales, int scale_layout, uint8_t *codes_t, int64_t ld_codes_t, uint8_t *scales_t,
                   int64_t ld_scales_t, void *stream) {
    Range range_("mxfp4_quantize");
    if (!x || !codes || !scales) return MXFP4_ERR_INVALID_ARG;
    if (rows <= 0 || cols <= 0) return MXFP4_ERR_INVALID_ARG;
    if (layout != MXFP4_LAYOUT_1D_ROW && layout != MXFP4_LAYOUT_1D_COL && layout != MXFP4_LAYOUT_2D)
        return MXFP4_ERR_INVALID_ARG;
    if (rht_size != 0 && rht_size != 16 && rht_size != 32) return MXFP4_ERR_INVALID_ARG;
    if (!valid_rounding(rounding)) return MXFP4_ERR_INVALID_ARG;
    if (scale_layout != MXFP4_SCALES_ROWMAJOR && scale_layout != MXFP4_SCALES_MMA) return MXFP4_ERR_INVALID_ARG;
    if ((elem_offset & 3u) != 0) return MXFP4_ERR_INVALID_ARG;
    if (layout == MXFP4_LAYOUT_1D_ROW && (cols % 32)) return MXFP4_ERR_INVALID_ARG;
    if (layout == MXFP4_LAYOUT_1D_COL && (rows % 32)) return MXFP4_ERR_INVALID_ARG;
    if (layout == MXFP4_LAYOUT_2D && ((rows % 32) || (cols % 32))) return MXFP4_ERR_INVALID_ARG;
    if (cols % 8) return MXFP4_ERR_INVALID_ARG;
    if ((codes_t || scales_t) && layout != MXFP4_LAYOUT_2D) return MXFP4_ERR_INVALID_ARG;
    if (scales_t && !codes_t) return MXFP4_ERR_INVALID_ARG;
    const int64_t code_cols = layout == MXFP4_LAYOUT_1D_COL ? rows / 2 : cols / 2;
    if (ld_x < cols || ld_codes < code_cols) return MXFP4_ERR_INVALID_ARG;
    if (scale_layout == MXFP4_SCALES_ROWMAJOR) {
        const int64_t sc = layout == MXFP4_LAYOUT_1D_COL ? rows / 32 : cols / 32;
        if (ld_scales < sc) return MXFP4_ERR_INVALID_ARG;
        if (scales_t && ld_scales_t < rows / 32) return MXFP4_ERR_INVALID_ARG;
    }
    if (codes_t && ld_codes_t < rows / 2) return MXFP4_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || (ld_x % 8) || (ld_codes % 16)) return MXFP4_ERR_ALIGNMENT;
    if (codes_t && (!aligned16(codes_t) || (ld_codes_t % 16))) return MXFP4_ERR_ALIGNMENT;
    if (scale_layout == MXFP4_SCALES_MMA && (!aligned16(scales) || (scales_t && !aligned16(scales_t))))
        return MXFP4_ERR_ALIGNMENT;
    const cudaError_t e = mxfp4::launch_quantize(x, rows, cols, ld_x, layout, rht_size, rounding, seed, elem_offset,
                                                 codes, ld_codes, scales, ld_scales, scale_layout, codes_t,
                                                 ld_codes_t, scales_t, ld_scales_t,
                                                 static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXFP4_OK : MXFP4_ERR_CUDA;
}

static int quantize_dual_impl(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int col_rht_size,
                              int rounding, uint64_t seed, uint64_t row_elem_offset, uint64_t col_elem_offset,
                              int64_t col_sr_ld, uint8_t *row_codes, int64_t ld_row_codes, uint8_t *row_scales,
                              int64_t ld_row_scales, uint8_t *col_codes, int64_t ld_col_codes, uint8_t *col_scales,
                              int64_t ld_col_scales, int scale_layout, void *stream);

int mxfp4_quantize_dual(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int col_rht_size, int rounding,
                        uint64_t seed, uint64_t row_elem_offset, uint64_t col_elem_offset, uint8_t *row_codes,
                        int64_t ld_row_codes, uint8_t *row_scales, int64_t ld_row_scales, uint8_t *col_codes,
                        int64_t ld_col_codes, uint8_t *col_scales, int64_t ld_col_scales, int scale_layout,
                        void *stream) {
    Range range_("mxfp4_quantize_dual");
    return quantize_dual_impl(x, rows, cols, ld_x, col_rht_size, rounding, seed, row_elem_offset, col_elem_offset,
                              rows, row_codes, ld_row_codes, row_scales, ld_row_scales, col_codes, ld_col_codes,
                              col_scales, ld_col_scales, scale_layout, stream);
}

int mxfp4_quantize_dual_rows(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int64_t row0,
                             int64_t total_rows, int col_rht_size, int rounding, uint64_t seed, uint8_t *row_codes,
                             int64_t ld_row_codes, uint8_t *row_scales, int64_t ld_row_scales, uint8_t *col_codes,
                             int64_t ld_col_codes, uint8_t *col_scales, int64_t ld_col_scales, int scale_layout,
                             void *stream) {
    Range range_("mxfp4_quantize_dual_rows");
    if (row0 < 0 || (row0 % 32) || total_rows <= 0 || (total_rows % 32) || rows > total_rows - row0)
        return MXFP4_ERR_INVALID_ARG;
    if (cols > 0 && row0 > ((int64_t)1 << 62) / cols) return MXFP4_ERR_UNSUPPORTED;
    // row output: rows of the whole tensor, offset row0 * cols; column output:
    // columns of the whole tensor's [cols, total_rows] view from column row0
    return quantize_dual_impl(x, rows, cols, ld_x, col_rht_size, rounding, seed, (uint64_t)(row0 * cols),
                              (uint64_t)row0, total_rows, row_codes, ld_row_codes, row_scales, ld_row_scales,
                              col_codes, ld_col_codes, col_scales, ld_col_scales, scale_layout, stream);
}

static int quantize_dual_impl(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int col_rht_size,
                              int rounding, uint64_t seed, uint64_t row_elem_offset, uint64_t col_elem_offset,
                              int64_t col_sr_ld, uint8_t *row_codes, int64_t ld_row_codes, uint8_t *row_scales,
                              int64_t ld_row_scales, uint8_t *col_codes, int64_t ld_col_codes, uint8_t *col_scales,
                              int64_t ld_col_scales, int scale_layout, void *stream) {
    if (!x || (!row_codes && !col_codes)) return MXFP4_ERR_INVALID_ARG;
    if ((row_codes && !row_scales) || (col_codes && !col_scales)) return MXFP4_ERR_INVALID_ARG;
    if (rows <= 0 || cols <= 0 || (rows % 32) || (cols % 32)) return MXFP4_ERR_INVALID_ARG;
    if (col_rht_size != 0 && col_rht_size != 16 && col_rht_size != 32) return MXFP4_ERR_INVALID_ARG;
    if (!valid_rounding(rounding)) return MXFP4_ERR_INVALID_ARG;
    if (scale_layout != MXFP4_SCALES_ROWMAJOR && scale_layout != MXFP4_SCALES_MMA) return MXFP4_ERR_INVALID_ARG;
    if ((row_elem_offset & 3u) || (col_elem_offset & 3u)) return MXFP4_ERR_INVALID_ARG;
    if (ld_x < cols) return MXFP4_ERR_INVALID_ARG;
    if (row_codes && ld_row_codes < cols / 2) return MXFP4_ERR_INVALID_ARG;
    if (col_codes && ld_col_codes < rows / 2) return MXFP4_ERR_INVALID_ARG;
    if (scale_layout == MXFP4_SCALES_ROWMAJOR) {
        if (row_codes && ld_row_scales < cols / 32) return MXFP4_ERR_INVALID_ARG;
        if (col_codes && ld_col_scales < rows / 32) return MXFP4_ERR_INVALID_ARG;
    }
    if (!aligned16(x) || (ld_x % 8)) return MXFP4_ERR_ALIGNMENT;
    if (row_codes && (!aligned16(row_codes) || (ld_row_codes % 16))) return MXFP4_ERR_ALIGNMENT;
    if (col_codes && (!aligned16(col_codes) || (ld_col_codes % 16))) return MXFP4_ERR_ALIGNMENT;
    // GEMM-ready scales are written in 4- and 16-byte pieces
    if (scale_layout == MXFP4_SCALES_MMA &&
        ((row_codes && !aligned16(row_scales)) || (col_codes && !aligned16(col_scales))))
        return MXFP4_ERR_ALIGNMENT;
    const cudaError_t e = mxfp4::launch_quantize_dual(
        x, rows, cols, ld_x, col_rht_size, rounding, seed, row_elem_offset, col_elem_offset, row_codes, ld_row_codes,
        row_scales, ld_row_scales, col_codes, ld_col_codes, col_scales, ld_col_scales, scale_layout, col_sr_ld,
        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXFP4_OK : MXFP4_ERR_CUDA;
}

int mxfp4_dequantize(const uint8_t *codes, int64_t ld_codes, const uint8_t *scales, int64_t ld_scales,
                     int scale_layout, int64_t rows, int64_t cols, int layout, int rht_size, uint64_t seed,
                     void *out, int64_t ld_out, int out_dtype, void *stream) {
    Range range_("mxfp4_dequantize");
    if (!codes || !scales || !out) return MXFP4_ERR_INVALID_ARG;
    if (rows <= 0 || cols <= 0) return MXFP4_ERR_INVALID_ARG;
    if (layout != MXFP4_LAYOUT_1D_ROW && layout != MXFP4_LAYOUT_1D_COL && layout != MXFP4_LAYOUT_2D)
        return MXFP4_ERR_INVALID_ARG;
    if (rht_size != 0 && rht_size != 16 && rht_size != 32) return MXFP4_ERR_INVALID_ARG;
    if (scale_layout != MXFP4_SCALES_ROWMAJOR && scale_layout != MXFP4_SCALES_MMA) return MXFP4_ERR_INVALID_ARG;
    if (out_dtype != MXFP4_OUT_BF16 && out_dtype != MXFP4_OUT_F32) return MXFP4_ERR_INVALID_ARG;
    if (layout == MXFP4_LAYOUT_1D_ROW && (cols % 32)) return MXFP4_ERR_INVALID_ARG;
    if (layout == MXFP4_LAYOUT_1D_COL && (rows % 32)) return MXFP4_ERR_INVALID_ARG;
    if (layout == MXFP4_LAYOUT_2D && ((rows % 32) || (cols % 32))) return MXFP4_ERR_INVALID_ARG;
    if (cols % 8) return MXFP4_ERR_INVALID_ARG;
    const int64_t code_cols = layout == MXFP4_LAYOUT_1D_COL ? rows / 2 : cols / 2;
    if (ld_codes < code_cols || ld_out < cols) return MXFP4_ERR_INVALID_ARG;
    if (scale_layout == MXFP4_SCALES_ROWMAJOR) {
        const int64_t sc = layout == MXFP4_LAYOUT_1D_COL ? rows / 32 : cols / 32;
        if (ld_scales < sc) return MXFP4_ERR_INVALID_ARG;
    }
    if (!aligned16(codes) || !aligned16(out) || (ld_codes % 16) || (ld_out % 8)) return MXFP4_ERR_ALIGNMENT;
    const cudaError_t e = mxfp4::launch_dequantize(codes, ld_codes, scales, ld_scales, scale_layout, rows, cols,
                                                   layout, rht_size, seed, out, ld_out, out_dtype,
                                                   static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXFP4_OK : MXFP4_ERR_CUDA;
}

// c_elem: bytes per output element (4 FP32, 2 bf16); TMA stores need 16-byte rows.
static int check_gemm_common(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes,
                             int64_t ldb, const uint8_t *b_scales, int64_t N, int64_t K, const void *c,
                             int64_t ldc, int c_elem = 4) {
    if (!a_codes || !a_scales || !b_codes || !b_scales || !c) return MXFP4_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0) return MXFP4_ERR_INVALID_ARG;
    if (K % 32) return MXFP4_ERR_INVALID_ARG;
    if (K % 64) return MXFP4_ERR_UNSUPPORTED;
    if (lda < K / 2 || ldb < K / 2 || ldc < N) return MXFP4_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(a_scales) || !aligned16(b_scales) ||
        !aligned16(c) || (lda % 16) || (ldb % 16) || ((ldc * c_elem) % 16))
        return MXFP4_ERR_ALIGNMENT;
    if (N > (int64_t)1 << 31 || K > (int64_t)1 << 31) return MXFP4_ERR_UNSUPPORTED;
    return MXFP4_OK;
}

int mxfp4_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes, int64_t ldb,
               const uint8_t *b_scales, int64_t M, int64_t N, int64_t K, float *c, int64_t ldc, void *stream) {
    Range range_("mxfp4_gemm");
    if (M <= 0) return MXFP4_ERR_INVALID_ARG;
    const int rc = check_gemm_common(a_codes, lda, a_scales, b_codes, ldb, b_scales, N, K, c, ldc);
    if (rc != MXFP4_OK) return rc;
    if (M > (int64_t)1 << 31) return MXFP4_ERR_UNSUPPORTED;
    return mxfp4::launch_gemm(a_codes, lda, a_scales, b_codes, ldb, b_scales, M, N, K, c, ldc,
                              static_cast<cudaStream_t>(stream));
}

int mxfp4_grouped_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, int64_t a_rows,
                       const int32_t *group_offsets, const int32_t *group_sizes, int num_groups,
                       const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales, int64_t N, int64_t K, float *c,
                       int64_t ldc, void *stream) {
    Range range_("mxfp4_grouped_gemm");
    if (!group_offsets || !group_sizes) return MXFP4_ERR_INVALID_ARG;
    if (num_groups <= 0 || a_rows <= 0) return MXFP4_ERR_INVALID_ARG;
    if (num_groups > 1024) return MXFP4_ERR_UNSUPPORTED;
    const int rc = check_gemm_common(a_codes, lda, a_scales, b_codes, ldb, b_scales, N, K, c, ldc);
    if (rc != MXFP4_OK) return rc;
    if (a_rows > (int64_t)1 << 31 || (int64_t)num_groups * N > (int64_t)1 << 31) return MXFP4_ERR_UNSUPPORTED;
    return mxfp4::launch_grouped_gemm(a_codes, lda, a_scales, a_rows, group_offsets, group_sizes, num_groups,
                                      b_codes, ldb, b_scales, N, K, c, ldc, static_cast<cudaStream_t>(stream));
}

int mxfp4_gemm_bf16(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes,
                    int64_t ldb, const uint8_t *b_scales, int64_t M, int64_t N, int64_t K, uint16_t *c, int64_t ldc,
                    void *stream) {
    Range range_("mxfp4_gemm_bf16");
    if (M <= 0) return MXFP4_ERR_INVALID_ARG;
    const int rc = check_gemm_common(a_codes, lda, a_scales, b_codes, ldb, b_scales, N, K, c, ldc, 2);
    if (rc != MXFP4_OK) return rc;
    if (M > (int64_t)1 << 31) return MXFP4_ERR_UNSUPPORTED;
    return mxfp4::launch_gemm_bf16(a_codes, lda, a_scales, b_codes, ldb, b_scales, M, N, K, c, ldc,
                                   static_cast<cudaStream_t>(stream));
}

int mxfp4_gemm_mxfp4(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes,
                     int64_t ldb, const uint8_t *b_scales, int64_t M, int64_t N, int64_t K, uint8_t *c_codes,
                     int64_t ld_c_codes, uint8_t *c_scales, int64_t ld_c_scales, int c_scale_layout, void *stream) {
    Range range_("mxfp4_gemm_mxfp4");
    if (!a_codes || !a_scales || !b_codes || !b_scales || !c_codes || !c_scales) return MXFP4_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0 || (N % 32) || (K % 32)) return MXFP4_ERR_INVALID_ARG;
    if (c_scale_layout != MXFP4_SCALES_ROWMAJOR && c_scale_layout != MXFP4_SCALES_MMA) return MXFP4_ERR_INVALID_ARG;
    if (K % 64) return MXFP4_ERR_UNSUPPORTED;
    if (lda < K / 2 || ldb < K / 2 || ld_c_codes < N / 2) return MXFP4_ERR_INVALID_ARG;
    if (c_scale_layout == MXFP4_SCALES_ROWMAJOR && ld_c_scales < N / 32) return MXFP4_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(a_scales) || !aligned16(b_scales) ||
        !aligned16(c_codes) || (lda % 16) || (ldb % 16) || (ld_c_codes % 16))
        return MXFP4_ERR_ALIGNMENT;
    if (M > (int64_t)1 << 31 || N > (int64_t)1 << 31 || K > (int64_t)1 << 31) return MXFP4_ERR_UNSUPPORTED;
    return mxfp4::launch_gemm_mx(a_codes, lda, a_scales, b_codes, ldb, b_scales, M, N, K, c_codes, ld_c_codes,
                                 c_scales, ld_c_scales, c_scale_layout == MXFP4_SCALES_MMA,
                                 static_cast<cudaStream_t>(stream));
}

int mxfp4_grouped_gemm_bf16(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, int64_t a_rows,
                            const int32_t *group_offsets, const int32_t *group_sizes, int num_groups,
                            const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales, int64_t N, int64_t K,
                            uint16_t *c, int64_t ldc, void *stream) {
    Range range_("mxfp4_grouped_gemm_bf16");
    if (!group_offsets || !group_sizes) return MXFP4_ERR_INVALID_ARG;
    if (num_groups <= 0 || a_rows <= 0) return MXFP4_ERR_INVALID_ARG;
    if (num_groups > 1024) return MXFP4_ERR_UNSUPPORTED;
    const int rc = check_gemm_common(a_codes, lda, a_scales, b_codes, ldb, b_scales, N, K, c, ldc, 2);
    if (rc != MXFP4_OK) return rc;
    if (a_rows > (int64_t)1 << 31 || (int64_t)num_groups * N > (int64_t)1 << 31) return MXFP4_ERR_UNSUPPORTED;
    return mxfp4::launch_grouped_gemm_bf16(a_codes, lda, a_scales, a_rows, group_offsets, group_sizes, num_groups,
                                           b_codes, ldb, b_scales, N, K, c, ldc, static_cast<cudaStream_t>(stream));
}

int mxfp4_grouped_gemm_wgrad(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes,
                             int64_t ldb, const uint8_t *b_scales, const int32_t *group_offsets, int num_groups,
                             int64_t M, int64_t N, int64_t K, float *c, int64_t ldc, void *stream) {
    Range range_("mxfp4_grouped_gemm_wgrad");
    if (!group_offsets || num_groups <= 0 || M <= 0) return MXFP4_ERR_INVALID_ARG;
    if (num_groups > 1024) return MXFP4_ERR_UNSUPPORTED;
    const int rc = check_gemm_common(a_codes, lda, a_scales, b_codes, ldb, b_scales, N, K, c, ldc);
    if (rc != MXFP4_OK) return rc;
    if (K % 128) return MXFP4_ERR_INVALID_ARG;
    if (M > (int64_t)1 << 31 || (int64_t)num_groups * M > (int64_t)1 << 31) return MXFP4_ERR_UNSUPPORTED;
    return mxfp4::launch_grouped_wgrad(a_codes, lda, a_scales, b_codes, ldb, b_scales, group_offsets, num_groups, M,
                                       N, K, c, ldc, static_cast<cudaStream_t>(stream));
}

int mxfp4_grouped_gemm_wgrad_bf16(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales,
                                  const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales,
                                  const int32_t *group_offsets, int num_groups, int64_t M, int64_t N, int64_t K,
                                  uint16_t *c, int64_t ldc, void *stream) {
    Range range_("mxfp4_grouped_gemm_wgrad_bf16");
    if (!group_offsets || num_groups <= 0 || M <= 0) return MXFP4_ERR_INVALID_ARG;
    if (num_groups > 1024) return MXFP4_ERR_UNSUPPORTED;
    const int rc = check_gemm_common(a_codes, lda, a_scales, b_codes, ldb, b_scales, N, K, c, ldc, 2);
    if (rc != MXFP4_OK) return rc;
    if (K % 128) return MXFP4_ERR_INVALID_ARG;
    if (M > (int64_t)1 << 31 || (int64_t)num_groups * M > (int64_t)1 << 31) return MXFP4_ERR_UNSUPPORTED;
    return mxfp4::launch_grouped_wgrad_bf16(a_codes, lda, a_scales, b_codes, ldb, b_scales, group_offsets,
                                            num_groups, M, N, K, c, ldc, static_cast<cudaStream_t>(stream));
}

int mxfp4_nvfp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int layout, int rounding,
                         uint64_t seed, uint64_t elem_offset, float *tensor_amax, uint8_t *codes, int64_t ld_codes,
                         uint8_t *scales, int64_t ld_scales, int scale_layout, void *stream) {
    Range range_("mxfp4_nvfp4_quantize");
    if (!x || !codes || !scales || !tensor_amax) return MXFP4_ERR_INVALID_ARG;
    if (rows <= 0 || cols <= 0) return MXFP4_ERR_INVALID_ARG;
    if (layout != MXFP4_LAYOUT_1D_ROW && layout != MXFP4_LAYOUT_1D_COL) return MXFP4_ERR_INVALID_ARG;
    if (rounding != MXFP4_ROUND_RNE && rounding != MXFP4_ROUND_SR) return MXFP4_ERR_INVALID_ARG;
    if (scale_layout != MXFP4_SCALES_ROWMAJOR && scale_layout != MXFP4_SCALES_MMA) return MXFP4_ERR_INVALID_ARG;
    const bool col = layout == MXFP4_LAYOUT_1D_COL;
    const int64_t orows = col ? cols : rows, k = col ? rows : cols;
    if (rows % 16 || cols % 16 || (elem_offset % 4)) return MXFP4_ERR_INVALID_ARG;
    if (ld_x < cols || ld_codes < k / 2) return MXFP4_ERR_INVALID_ARG;
    if (scale_layout == MXFP4_SCALES_ROWMAJOR && ld_scales < k / 16) return MXFP4_ERR_INVALID_ARG;
    if (!aligned16(x) || (ld_x % 8) || !aligned16(codes) || (ld_codes % 16) ||
        (reinterpret_cast<uintptr_t>(tensor_amax) & 3u))
        return MXFP4_ERR_ALIGNMENT;
    if (orows > (int64_t)1 << 31 || k > (int64_t)1 << 31) return MXFP4_ERR_UNSUPPORTED;
    const cudaError_t e = mxfp4::launch_nvfp4_quantize(x, rows, cols, ld_x, layout, rounding, seed, elem_offset,
                                                       tensor_amax, codes, ld_codes, scales, ld_scales, scale_layout,
                                                       static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXFP4_OK : MXFP4_ERR_CUDA;
}

int mxfp4_nvfp4_dequantize(const uint8_t *codes, int64_t ld_codes, const uint8_t *scales, int64_t ld_scales,
                           int scale_layout, const float *tensor_amax, int64_t rows, int64_t cols, int layout,
                           float *out, int64_t ld_out, void *stream) {
    Range range_("mxfp4_nvfp4_dequantize");
    if (!codes || !scales || !tensor_amax || !out) return MXFP4_ERR_INVALID_ARG;
    if (rows <= 0 || cols <= 0 || rows % 16 || cols % 16) return MXFP4_ERR_INVALID_ARG;
    if (layout != MXFP4_LAYOUT_1D_ROW && layout != MXFP4_LAYOUT_1D_COL) return MXFP4_ERR_INVALID_ARG;
    if (scale_layout != MXFP4_SCALES_ROWMAJOR && scale_layout != MXFP4_SCALES_MMA) return MXFP4_ERR_INVALID_ARG;
    const bool col = layout == MXFP4_LAYOUT_1D_COL;
    const int64_t k = col ? rows : cols;
    if (ld_codes < k / 2 || ld_out < cols) return MXFP4_ERR_INVALID_ARG;
    if (scale_layout == MXFP4_SCALES_ROWMAJOR && ld_scales < k / 16) return MXFP4_ERR_INVALID_ARG;
    if ((ld_codes % 8) || (reinterpret_cast<uintptr_t>(codes) & 7u) || !aligned16(out) || (ld_out % 4))
        return MXFP4_ERR_ALIGNMENT;
    const cudaError_t e = mxfp4::launch_nvfp4_dequantize(codes, ld_codes, scales, ld_scales, scale_layout,
                                                         tensor_amax, rows, cols, layout, out, ld_out,
                                                         static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXFP4_OK : MXFP4_ERR_CUDA;
}

int mxfp4_nvfp4_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const float *a_amax,
                     const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales, const float *b_amax, int64_t M,
                     int64_t N, int64_t K, float *c, int64_t ldc, void *stream) {
    Range range_("mxfp4_nvfp4_gemm");
    if (M <= 0 || !a_amax || !b_amax) return MXFP4_ERR_INVALID_ARG;
    const int rc = check_gemm_common(a_codes, lda, a_scales, b_codes, ldb, b_scales, N, K, c, ldc);
    if (rc != MXFP4_OK) return rc;
    if (M > (int64_t)1 << 31) return MXFP4_ERR_UNSUPPORTED;
    return mxfp4::launch_nvfp4_gemm(a_codes, lda, a_scales, a_amax, b_codes, ldb, b_scales, b_amax, M, N, K, c, ldc,
                                    static_cast<cudaStream_t>(stream));
}

int mxfp4_scales_to_mma(const uint8_t *scales, int64_t ld_scales, int64_t rows, int64_t k, int two_d,
                        uint8_t *mma_scales, void *stream) {
    Range range_("mxfp4_scales_to_mma");
    if (!scales || !mma_scales) return MXFP4_ERR_INVALID_ARG;
    if (rows <= 0 || k <= 0 || (k % 32) || (two_d != 0 && two_d != 1)) return MXFP4_ERR_INVALID_ARG;
    if (two_d && (rows % 32)) return MXFP4_ERR_INVALID_ARG;
    if (ld_scales < k / 32) return MXFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(mma_scales) & 3u) != 0) return MXFP4_ERR_ALIGNMENT;
    if (rows > (int64_t)1 << 40 || k > (int64_t)1 << 40) return MXFP4_ERR_UNSUPPORTED;
    const cudaError_t e = mxfp4::launch_scales_to_mma(scales, ld_scales, rows, k, two_d, mma_scales,
                                                      static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXFP4_OK : MXFP4_ERR_CUDA;
}

int mxfp4_get_error(void *stream) { return mxfp4::get_error(static_cast<cudaStream_t>(stream)); }

uint64_t mxfp4_set_wait_limit_ns(uint64_t limit_ns) { return mxfp4::set_wait_limit(limit_ns); }

int mxfp4_wait_probe(int arrive, void *stream) {
    Range range_("mxfp4_wait_probe");
    return mxfp4::launch_wait_probe(arrive, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
