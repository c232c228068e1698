// nvfp4.cu -- NVFP4 quantize and dequantize for sm_100a.
//
// "MXFP4" (aiwiki.ai), "Comparison with NVFP4": E2M1 elements in blocks of 16,
// an FP8 E4M3 block scale fitted to each block, and a second-level FP32 scale
// per tensor (4.5 bits per value).  The page gives the format, not the scale
// rule; the rule implemented here:
//   S = fp32(amax_tensor / 2688)            (2688 = 6 * 448: the largest block
//                                            scale is E4M3's maximum)
//   block code = E4M3 nearest-even of fp32(amax_block / fp32(6 S)),
//                saturating at 448
//   X = fp32(decode(code) * S); elements fp32(x / X) to E2M1 (nearest-even
//   with saturation, or stochastic rounding with the Philox stream of the
//   MXFP4 quantizer).  A block whose scale rounds to 0 stores +-0; a NaN or
//   Inf in the tensor gives every block the NaN scale 0x7F and zero codes.
// The tensor amax is computed on the device first (into the caller's float),
// so quantization needs no host synchronization; the GEMM reads the same
// float for its epilogue.
#include <cstdint>
#include <cstring>

#include "common.cuh"

namespace mxfp4 {

struct NvParams {
    const uint16_t *x;
    int64_t rows, cols, ld_x;
    uint8_t *codes, *scales;
    int64_t ld_codes, ld_scales, katoms;   // katoms: MMA-layout atoms (4 blocks of 16) along K
    const uint32_t *amax_bits;             // tensor amax as fp32 bits (written by nv_amax_kernel)
    uint32_t seed_lo, seed_hi;
    uint64_t elem_offset;
};

__device__ __forceinline__ uint4 nv_ldg_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// E4M3 byte (finite) -> fp32, exact: (1 + m/8) 2^(e-7), or m 2^-9 when e = 0.
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    const float v = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
    return (c & 0x80u) ? -v : v;
}

// Nearest-even E4M3 of q >= 0, saturating at 448 (NaN -> 0x7F).
__device__ __forceinline__ uint32_t f32_to_e4m3(float q) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(0.0f), "f"(q));
    return d & 0xFFu;
}

// ---------------------------------------------------------------------------
// Tensor amax: the largest bf16 magnitude, NaN if any element is NaN.  As
// unsigned integers the magnitude bit patterns order like the values, with
// Inf above every finite value and NaN above Inf, so one integer max suffices.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) nv_amax_kernel(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld_x,
                                                      uint32_t *amax_bits) {
    pdl_wait();
    pdl_trigger();
    uint32_t m = 0;
    const int64_t chunks = cols / 8, n = rows * chunks;
    // (row, chunk) of the flat index i, stepped by the grid stride without a
    // division per iteration
    const int64_t i0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x, stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t dr = stride / chunks, dc = stride - dr * chunks;
    int64_t r = i0 / chunks, ch = i0 - r * chunks;
    auto step = [&]() {
        r += dr;
        ch += dc;
        if (ch >= chunks) { ch -= chunks; ++r; }
    };
    // two loads in flight per thread
    for (int64_t i = i0; i < n; i += 2 * stride) {
        const uint4 u = nv_ldg_v4(x + r * ld_x + 8 * ch);
        step();
        uint4 v = make_uint4(0, 0, 0, 0);
        if (i + stride < n) v = nv_ldg_v4(x + r * ld_x + 8 * ch);
        step();
        const uint32_t w[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) m = max(m, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0 && m) atomicMax(amax_bits, m << 16);
}

// Tensor scale from the device amax; `bad` for a NaN or Inf tensor.
struct NvTensor {
    float S, six_s;
    bool bad;
};
__device__ __forceinline__ NvTensor nv_tensor(const uint32_t *amax_bits) {
    NvTensor t;
    const float amax = __uint_as_float(*amax_bits);
    t.bad = !(amax <= 3.4028234664e38f);
    t.S = __fdiv_rn(amax, 2688.0f);
    t.six_s = __fmul_rn(6.0f, t.S);
    return t;
}

// One block of 16 values -> scale code and 8 bytes of element codes.
// g0: stream index of element 0 (a multiple of 4).
template <bool SR>
__device__ __forceinline__ uint32_t nv_block(float *v, const NvTensor &t, uint64_t g0, uint32_t k0, uint32_t k1,
                                             uint2 &out) {
    if (t.bad) {
        out = make_uint2(0, 0);
        return 0x7Fu;
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const uint32_t code = t.S > 0.0f ? f32_to_e4m3(__fdiv_rn(amax, t.six_s)) : 0u;
    const float X = __fmul_rn(e4m3_to_f32(code), t.S);
    if (X == 0.0f) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = copysignf(0.0f, v[i]);
    } else {
        // The quotients v / X rounded to nearest even.  With y = RN(1/X),
        // q = RN(|v| y) is within one ulp of |v| / X, the residual |v| - q X
        // is exact by FMA, and RN(q + (|v| - q X) y) is the correctly rounded
        // quotient (Markstein's FMA division, "Computation of elementary
        // functions on the IBM RISC System/6000 processor", 1990); the sign
        // goes back on exactly.  The residual must not underflow and the
        // reciprocal must be normal, so the block takes this path only when
        // X lies in [2^-100, 2^100] and every nonzero |v| is at least 2^-100
        // (the quotients are below 16 here); otherwise each element is
        // divided with the IEEE division.
        bool tiny = !(X >= 0x1p-100f && X <= 0x1p100f);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float a = fabsf(v[i]);
            tiny |= a != 0.0f && a < 0x1p-100f;
        }
        if (!tiny) {
            const float y = __frcp_rn(X);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float a = fabsf(v[i]);
                const float q = __fmul_rn(a, y);
                const float r = __fmaf_rn(-q, X, a);
                v[i] = copysignf(__fmaf_rn(r, y, q), v[i]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = __fdiv_rn(v[i], X);
        }
    }
    if constexpr (!SR) {
        out = make_uint2(e2m1x8_rn(v), e2m1x8_rn(v + 8));
    } else {
        const uint64_t blk = g0 >> 2;
        uint32_t p[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            p[q] = e2m1x8_sr(v + 8 * q, blk + 2 * q, k0, k1);
        }
        out = make_uint2(p[0], p[1]);
    }
    return code;
}

__device__ __forceinline__ void nv_store_scale(const NvParams &p, bool mma, int64_t row, int64_t kb, uint32_t code) {
    if (mma) p.scales[mma_scale_off(row, kb, p.katoms)] = (uint8_t)code;
    else p.scales[row * p.ld_scales + kb] = (uint8_t)code;
}

// Row blocks: one thread per block of 16 (32 bytes of input).
template <bool SR, bool MMA>
__global__ void __launch_bounds__(256) nv_quant_row_kernel(const NvParams p) {
    pdl_wait();
    pdl_trigger();
    const NvTensor t = nv_tensor(p.amax_bits);
    const int64_t nb = p.cols / 16, n = p.rows * nb;
    // (row, block) of the flat index i, stepped by the grid stride without a
    // division per iteration
    const int64_t i0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x, stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t dr = stride / nb, dk = stride - dr * nb;
    int64_t rr = i0 / nb, kk = i0 - rr * nb;
    // the next step's 32 bytes are loaded before this step's block is
    // quantized, so each thread keeps a load in flight through its compute
    uint4 u0 = make_uint4(0, 0, 0, 0), u1 = u0;
    if (i0 < n) {
        const uint16_t *src = p.x + rr * p.ld_x + 16 * kk;
        u0 = nv_ldg_v4(src);
        u1 = nv_ldg_v4(src + 8);
    }
    for (int64_t i = i0; i < n; i += stride) {
        const int64_t r = rr, kb = kk;
        rr += dr;
        kk += dk;
        if (kk >= nb) { kk -= nb; ++rr; }
        uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
        if (i + stride < n) {
            const uint16_t *src = p.x + rr * p.ld_x + 16 * kk;
            n0 = nv_ldg_v4(src);
            n1 = nv_ldg_v4(src + 8);
        }
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        u0 = n0;
        u1 = n1;
        float v[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) { v[2 * j] = bf16lo(w[j]); v[2 * j + 1] = bf16hi(w[j]); }
        uint2 q;
        const uint32_t code = nv_block<SR>(v, t, (uint64_t)(r * p.cols + 16 * kb) + p.elem_offset, p.seed_lo,
                                           p.seed_hi, q);
        *reinterpret_cast<uint2 *>(p.codes + r * p.ld_codes + 8 * kb) = q;
        nv_store_scale(p, MMA, r, kb, code);
    }
}

// Column blocks (transposed output): 64 x 64 tiles through shared memory;
// thread (column c, block b) quantizes rows 16b..16b+15 of column c; the
// codes are staged so that each output row leaves as 32 contiguous bytes.
constexpr int NV_T = 64, NV_PITCH = NV_T + 8;

template <bool SR, bool MMA>
__global__ void __launch_bounds__(256) nv_quant_col_kernel(const NvParams p) {
    pdl_wait();
    pdl_trigger();
    __shared__ __align__(16) uint16_t tin[NV_T * NV_PITCH];
    __shared__ __align__(16) uint2 tout[NV_T][4];
    const int tid = threadIdx.x;
    const NvTensor t = nv_tensor(p.amax_bits);
    const int64_t tiles_c = (p.cols + NV_T - 1) / NV_T, tiles = ((p.rows + NV_T - 1) / NV_T) * tiles_c;
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int64_t r0 = (tile / tiles_c) * NV_T, c0 = (tile % tiles_c) * NV_T;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int idx = tid + 256 * i, row = idx >> 3, ch = idx & 7;
            const int64_t gr = r0 + row, gc = c0 + 8 * ch;
            if (gr < p.rows && gc < p.cols)
                *reinterpret_cast<uint4 *>(tin + row * NV_PITCH + 8 * ch) = nv_ldg_v4(p.x + gr * p.ld_x + gc);
        }
        __syncthreads();
        const int c = tid & 63, b = tid >> 6;
        const int64_t orow = c0 + c, rin = r0 + 16 * b;
        if (orow < p.cols && rin < p.rows) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = __uint_as_float((uint32_t)tin[(16 * b + i) * NV_PITCH + c] << 16);
            uint2 q;
            const uint32_t code = nv_block<SR>(v, t, (uint64_t)(orow * p.rows + rin) + p.elem_offset, p.seed_lo,
                                               p.seed_hi, q);
            tout[c][b] = q;
            nv_store_scale(p, MMA, orow, rin >> 4, code);
        }
        __syncthreads();
        if (tid < 128) {
            const int row = tid >> 1, half = tid & 1;           // 32 bytes per output row, 16 per thread
            const int64_t orow2 = c0 + row, rin2 = r0 + 32 * half;
            if (orow2 < p.cols && rin2 < p.rows) {
                const uint2 a = tout[row][2 * half], bq = tout[row][2 * half + 1];
                if (rin2 + 16 < p.rows)
                    *reinterpret_cast<uint4 *>(p.codes + orow2 * p.ld_codes + (rin2 >> 1)) =
                        make_uint4(a.x, a.y, bq.x, bq.y);
                else
                    *reinterpret_cast<uint2 *>(p.codes + orow2 * p.ld_codes + (rin2 >> 1)) = a;
            }
        }
        __syncthreads();
    }
}

struct NvDeqParams {
    const uint8_t *codes, *scales;
    int64_t ld_codes, ld_scales, katoms;
    int64_t rows, cols;                    // the dequantized tensor
    float *out;
    int64_t ld_out;
    const uint32_t *amax_bits;
};

// One thread per block of 16: value = fp32(fp32(code * scale) * S).
template <bool COL, bool MMA>
__global__ void __launch_bounds__(256) nv_dequant_kernel(const NvDeqParams p) {
    pdl_wait();
    pdl_trigger();
    const float S = __fdiv_rn(__uint_as_float(*p.amax_bits), 2688.0f);
    const int64_t orows = COL ? p.cols : p.rows, k = COL ? p.rows : p.cols;
    const int64_t nb = k / 16, n = orows * nb;
    // (output row, block) of the flat index i, stepped by the grid stride
    const int64_t i0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x, stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t dr = stride / nb, dk = stride - dr * nb;
    int64_t rr = i0 / nb, kk = i0 - rr * nb;
    for (int64_t i = i0; i < n; i += stride) {
        const int64_t orow = rr, kb = kk;
        rr += dr;
        kk += dk;
        if (kk >= nb) { kk -= nb; ++rr; }
        const uint32_t sc = MMA ? p.scales[mma_scale_off(orow, kb, p.katoms)] : p.scales[orow * p.ld_scales + kb];
        const bool nan = (sc & 0x7Fu) == 0x7Fu;
        const float s = nan ? __uint_as_float(0x7FC00000u) : e4m3_to_f32(sc);
        const uint2 q = *reinterpret_cast<const uint2 *>(p.codes + orow * p.ld_codes + 8 * kb);
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint32_t nib = ((j < 8 ? q.x : q.y) >> (4 * (j & 7))) & 0xFu;
            v[j] = __fmul_rn(__fmul_rn(e2m1_value(nib), s), S);
        }
        if constexpr (!COL) {
            float4 *dst = reinterpret_cast<float4 *>(p.out + orow * p.ld_out + 16 * kb);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) p.out[(16 * kb + j) * p.ld_out + orow] = v[j];
        }
    }
}

static int nv_num_sms() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

static unsigned nv_grid(int64_t work) {
    const int64_t cap = (int64_t)nv_num_sms() * 16;
    const int64_t g = (work + 255) / 256;
    return (unsigned)(g < 1 ? 1 : (g > cap ? cap : g));
}

cudaError_t launch_nvfp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int layout, int rounding,
                                  uint64_t seed, uint64_t elem_offset, float *tensor_amax, uint8_t *codes,
                                  int64_t ld_codes, uint8_t *scales, int64_t ld_scales, int scale_layout,
                                  cudaStream_t s) {
    uint32_t *amax_bits = reinterpret_cast<uint32_t *>(tensor_amax);
    cudaError_t e = cudaMemsetAsync(amax_bits, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    e = launch_pdl(nv_amax_kernel, dim3(nv_grid(rows * (cols / 8))), dim3(256), 0, s,
                   static_cast<const uint16_t *>(x), rows, cols, ld_x, amax_bits);
    if (e != cudaSuccess) return e;
    NvParams p{};
    p.x = static_cast<const uint16_t *>(x);
    p.rows = rows; p.cols = cols; p.ld_x = ld_x;
    p.codes = codes; p.scales = scales; p.ld_codes = ld_codes; p.ld_scales = ld_scales;
    const int64_t k = layout == MXFP4_LAYOUT_1D_COL ? rows : cols;
    p.katoms = (k / 16 + 3) / 4;
    p.amax_bits = amax_bits;
    p.seed_lo = (uint32_t)seed; p.seed_hi = (uint32_t)(seed >> 32);
    p.elem_offset = elem_offset;
    const bool sr = (rounding & 0x0F) == MXFP4_ROUND_SR, mma = scale_layout == MXFP4_SCALES_MMA;
    if (layout == MXFP4_LAYOUT_1D_COL) {
        const int64_t tiles = ((rows + NV_T - 1) / NV_T) * ((cols + NV_T - 1) / NV_T);
        const unsigned g = (unsigned)(tiles < (int64_t)nv_num_sms() * 8 ? tiles : (int64_t)nv_num_sms() * 8);
        if (sr) return mma ? launch_pdl(nv_quant_col_kernel<true, true>, dim3(g), dim3(256), 0, s, p)
                           : launch_pdl(nv_quant_col_kernel<true, false>, dim3(g), dim3(256), 0, s, p);
        return mma ? launch_pdl(nv_quant_col_kernel<false, true>, dim3(g), dim3(256), 0, s, p)
                   : launch_pdl(nv_quant_col_kernel<false, false>, dim3(g), dim3(256), 0, s, p);
    }
    const unsigned g = nv_grid(rows * (cols / 16));
    if (sr) return mma ? launch_pdl(nv_quant_row_kernel<true, true>, dim3(g), dim3(256), 0, s, p)
                       : launch_pdl(nv_quant_row_kernel<true, false>, dim3(g), dim3(256), 0, s, p);
    return mma ? launch_pdl(nv_quant_row_kernel<false, true>, dim3(g), dim3(256), 0, s, p)
               : launch_pdl(nv_quant_row_kernel<false, false>, dim3(g), dim3(256), 0, s, p);
}

cudaError_t launch_nvfp4_dequantize(const uint8_t *codes, int64_t ld_codes, const uint8_t *scales, int64_t ld_scales,
                                    int scale_layout, const float *tensor_amax, int64_t rows, int64_t cols,
                                    int layout, float *out, int64_t ld_out, cudaStream_t s) {
    NvDeqParams p{};
    p.codes = codes; p.scales = scales; p.ld_codes = ld_codes; p.ld_scales = ld_scales;
    const bool col = layout == MXFP4_LAYOUT_1D_COL, mma = scale_layout == MXFP4_SCALES_MMA;
    const int64_t k = col ? rows : cols, orows = col ? cols : rows;
    p.katoms = (k / 16 + 3) / 4;
    p.rows = rows; p.cols = cols; p.out = out; p.ld_out = ld_out;
    p.amax_bits = reinterpret_cast<const uint32_t *>(tensor_amax);
    const unsigned g = nv_grid(orows * (k / 16));
    if (col) return mma ? launch_pdl(nv_dequant_kernel<true, true>, dim3(g), dim3(256), 0, s, p)
                        : launch_pdl(nv_dequant_kernel<true, false>, dim3(g), dim3(256), 0, s, p);
    return mma ? launch_pdl(nv_dequant_kernel<false, true>, dim3(g), dim3(256), 0, s, p)
               : launch_pdl(nv_dequant_kernel<false, false>, dim3(g), dim3(256), 0, s, p);
}

}  // namespace mxfp4
