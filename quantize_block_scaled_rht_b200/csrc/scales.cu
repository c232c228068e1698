// scales.cu -- canonical row-major E8M0 scales to the GEMM-ready layout.
//
// "MXFP4" (aiwiki.ai), "Use in models / gpt-oss": scales are stored apart from
// the element codes, one byte per 32-element block.  The canonical storage is
// row-major: [rows, k/32] for 1D blocks, or [rows/32, k/32] tile scales for
// 2D 32 x 32 blocks.  The block-scaled MMA reads its scale factors from
// tensor memory after a 32x128-bit copy of 512-byte atoms (128 rows x 4
// K-blocks, byte (row % 32) * 16 + ((row % 128) / 32) * 4 + kb % 4), so the
// GEMM takes that layout; this kernel produces it from the canonical one.
//
// One thread writes one 32-bit word of the output: the 4 K-blocks of one row
// in one atom.  Pad rows (to a multiple of 128) and pad K-blocks (to a
// multiple of 4) are written as zero, so the output is fully defined.
#include <cstdint>

#include <cuda_runtime.h>

#include "common.cuh"

namespace mxfp4 {

__global__ void __launch_bounds__(256) scales_to_mma_kernel(const uint8_t *__restrict__ src, int64_t ld_src,
                                                            int64_t rows, int64_t kblocks, int two_d,
                                                            uint32_t *__restrict__ dst, int64_t rows_pad,
                                                            int64_t katoms) {
    pdl_wait();
    pdl_trigger();
    const int64_t words = rows_pad * katoms;
    for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words;
         w += (int64_t)gridDim.x * blockDim.x) {
        // word w of the output, in output order: atom (row tile, katom), then
        // the 128 words of the atom at (row % 32) * 4 + (row % 128) / 32
        const int64_t atom = w >> 7;
        const int within = (int)(w & 127);
        const int64_t rt = atom / katoms, ka = atom - rt * katoms;
        const int64_t row = rt * 128 + (within & 3) * 32 + (within >> 2);
        uint32_t v = 0;
        if (row < rows) {
            const uint8_t *s = src + (two_d ? row / 32 : row) * ld_src;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t kb = ka * 4 + j;
                if (kb < kblocks) v |= (uint32_t)s[kb] << (8 * j);
            }
        }
        dst[w] = v;
    }
}

cudaError_t launch_scales_to_mma(const uint8_t *src, int64_t ld_src, int64_t rows, int64_t k, int two_d,
                                 uint8_t *dst, cudaStream_t s) {
    const int64_t katoms = mma_katoms(k), rows_pad = (rows + 127) / 128 * 128;
    const int64_t words = rows_pad * katoms;
    int64_t blocks = (words + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    return launch_pdl(scales_to_mma_kernel, dim3((unsigned)blocks), dim3(256), 0, s, src, ld_src, rows, k / 32,
                      two_d, reinterpret_cast<uint32_t *>(dst), rows_pad, katoms);
}

}  // namespace mxfp4
