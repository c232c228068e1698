// quantize.cu -- MXFP4 quantize / dequantize kernels for sm_100a.
//
// "MXFP4" (aiwiki.ai): "Format specification" (E2M1 codes, E8M0 scales,
// 32-element blocks), "Conversion rules" (X = 2^floor(log2 amax) / 4, RNE with
// saturation), "Training with MXFP4" (random Hadamard transform of size 16/32,
// stochastic rounding).  "Training an MoE LLM in MXFP4" (ALTO), abstract:
// 1D blocks for activations/gradients, 2D blocks for weights.
//
// Streaming kernels (2 B read + 0.5 B + 1/32 B written per element):
// 128-bit loads/stores, in-register Hadamard butterflies on packed two-lane
// fp32, and shared-memory staging only where a transpose is needed.  Under
// RNE they are bound by HBM; stochastic rounding adds the integer work of
// Philox4x32-10 and the exact rounding decision, which then bounds them.
#include <cstdint>
#include <map>
#include <mutex>
#include <cstdio>

#include "common.cuh"

namespace mxfp4 {

struct QuantParams {
    const uint16_t *x;
    int64_t rows, cols, ld_x;
    uint8_t *codes;
    int64_t ld_codes;
    uint8_t *scales;
    int64_t ld_scales, katoms;      // katoms: MMA layout K-atoms of the output operand
    uint8_t *codes_t;
    int64_t ld_codes_t;
    uint8_t *scales_t;
    int64_t ld_scales_t, katoms_t;
    uint32_t seed_lo, seed_hi;
    int scale_rule;                        // MXFP4_SCALE_* >> 4
    uint64_t elem_offset;
    // RHT signs as xor words: pair[j] flips the bf16 halves of word j of a
    // 32-element row segment (elements 2j, 2j+1); dup[i] flips both halves of
    // a word for element i of a column segment.
    uint32_t sgn_pair[16];
    uint32_t sgn_bit[32];                  // RHT sign of element i (mod the RHT size) as bit 31
};

// Packed two-lane fp32 arithmetic (sm_100a `.f32x2`): each lane is rounded
// to nearest even exactly as the scalar operation, subnormals kept.
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "sub.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// ---------------------------------------------------------------------------
// Per-block quantization core: the scale code from the block's amax, then the
// four groups of 8 values (unscaled, from get8(q, w)) scaled and encoded into
// 16 bytes of codes.  `g0` is the stream index of element 0.
// ---------------------------------------------------------------------------
template <bool SR, class Get8>
__device__ __forceinline__ uint32_t quantize_groups(float amax, Get8 &&get8, uint4 &out, uint64_t g0, uint32_t k0,
                                                    uint32_t k1, int rule) {
    const uint32_t code = scale_code_rule(amax, rule);
    if (code == 0xFFu) {
        out = make_uint4(0, 0, 0, 0);
        return code;
    }
    const float inv = inv_scale_from_code(code);
    const uint64_t blk = g0 >> 2;  // g0 % 4 == 0
    uint32_t p[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float w[8];
        get8(q, w);
        scale8(w, inv, rule);
        if constexpr (SR) p[q] = e2m1x8_sr(w, blk + 2 * q, k0, k1);
        else p[q] = e2m1x8_rn(w);
    }
    out = make_uint4(p[0], p[1], p[2], p[3]);
    return code;
}

// The same for 32 fp32 values already in registers (transformed if the RHT
// applies).
template <bool SR>
__device__ __forceinline__ uint32_t quantize32(const float *v, uint4 &out, uint64_t g0, uint32_t k0, uint32_t k1,
                                           int rule) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; i += 2) amax = amax_nan2(amax, v[i], v[i + 1]);
    return quantize_groups<SR>(
        amax,
        [&](int q, float *w) {
#pragma unroll
            for (int j = 0; j < 8; ++j) w[j] = v[8 * q + j];
        },
        out, g0, k0, k1, rule);
}

// The same butterfly as fwht<D> on 32 values held as 16 pairs
// P[m] = (v[m], v[m + 16]).  Stages h = 1, 2, 4, 8 act on both 16-element
// halves at once (the two lanes of a pair), with the same operations in the
// same order; for D = 32 the last stage (h = 16) combines the two lanes of
// each pair.  Bit-identical to fwht<D> on v (both halves for D = 16).
template <int D>
__device__ __forceinline__ void fwht_pairs(float2 *P) {
    static_assert(D == 16 || D == 32, "RHT size");
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            if ((m & h) == 0) {
                const float2 a = P[m], b = P[m + h];
                P[m] = add2(a, b);
                P[m + h] = sub2(a, b);
            }
        }
    }
    if constexpr (D == 32) {
#pragma unroll
        for (int m = 0; m < 16; ++m) P[m] = make_float2(__fadd_rn(P[m].x, P[m].y), __fsub_rn(P[m].x, P[m].y));
    }
}

// fwht<D> on v[0..31] (each D-element segment) followed by the product with
// c, through the packed pairs (v[m], v[m + 16]); bit-identical to the scalar
// loops.
template <int D>
__device__ __forceinline__ void fwht32_scaled(float *v, float c) {
    float2 P[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) P[m] = make_float2(v[m], v[m + 16]);
    fwht_pairs<D>(P);
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        P[m] = mul2(P[m], make_float2(c, c));
        v[m] = P[m].x;
        v[m + 16] = P[m].y;
    }
}

// The same for 32 fp32 values held as 16 pairs P[m] = (v[m], v[m + 16]),
// scaled with packed two-lane multiplies (each lane rounded as the scalar
// product): groups 0, 1 are the low lanes of P[0..15], groups 2, 3 the high.
__device__ __forceinline__ float amax_pairs(const float2 *P) {
    float amax = 0.0f;
#pragma unroll
    for (int m = 0; m < 16; ++m) amax = amax_nan2(amax, P[m].x, P[m].y);
    return amax;
}

// The block's scale from a given amax (a 2D tile's, or the block's own) and
// the elements from the pairs.
template <bool SR>
__device__ __forceinline__ uint32_t quantize32_pairs_amax(float2 *P, float amax, uint4 &out, uint64_t g0,
                                                          uint32_t k0, uint32_t k1, int rule) {
    const uint32_t code = scale_code_rule(amax, rule);
    if (code == 0xFFu) {
        out = make_uint4(0, 0, 0, 0);
        return code;
    }
    const float inv = inv_scale_from_code(code);
    if (rule == 2) {
#pragma unroll
        for (int m = 0; m < 16; ++m) P[m] = mul2(mul2(P[m], make_float2(0.75f, 0.75f)), make_float2(inv, inv));
    } else {
#pragma unroll
        for (int m = 0; m < 16; ++m) P[m] = mul2(P[m], make_float2(inv, inv));
    }
    const uint64_t blk = g0 >> 2;  // g0 % 4 == 0
    uint32_t p[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = q < 2 ? P[8 * q + j].x : P[8 * (q - 2) + j].y;
        if constexpr (SR) p[q] = e2m1x8_sr(w, blk + 2 * q, k0, k1);
        else p[q] = e2m1x8_rn(w);
    }
    out = make_uint4(p[0], p[1], p[2], p[3]);
    return code;
}

template <bool SR>
__device__ __forceinline__ uint32_t quantize32_pairs(float2 *P, uint4 &out, uint64_t g0, uint32_t k0, uint32_t k1,
                                                     int rule) {
    return quantize32_pairs_amax<SR>(P, amax_pairs(P), out, g0, k0, k1, rule);
}

// The same for 32 bf16 values packed in four uint4 (no transform): amax on
// the packed pairs, each group unpacked when it is encoded, so that the block
// occupies 16 registers rather than 32.
template <bool SR>
__device__ __forceinline__ uint32_t quantize32_bf16(const uint4 *u, uint4 &out, uint64_t g0, uint32_t k0, uint32_t k1,
                                                int rule) {
    return quantize_groups<SR>(
        amax_bf16x32(u), [&](int q, float *w) { unpack_bf16x8(u[q], w); }, out, g0, k0, k1, rule);
}

// Unpack 16 bf16x2 words to 32 fp32 values, with RHT sign flips and butterfly.
// A row block of 32 bf16 values (w[j]: elements 2j, 2j + 1) as the pairs
// P[m] = (v[m], v[m + 16]) of the packed butterfly, sign-flipped, transformed
// and normalised; the same values as unpack_row32.
template <int RHT>
__device__ __forceinline__ void unpack_row32_pairs(const uint32_t *w, float2 *P, const QuantParams &p) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t a = w[j] ^ p.sgn_pair[j], b = w[j + 8] ^ p.sgn_pair[j + 8];
        P[2 * j] = make_float2(bf16lo(a), bf16lo(b));
        P[2 * j + 1] = make_float2(bf16hi(a), bf16hi(b));
    }
    const float c = rht_norm<RHT>();
    fwht_pairs<RHT>(P);
#pragma unroll
    for (int m = 0; m < 16; ++m) P[m] = mul2(P[m], make_float2(c, c));
}

template <int RHT>
__device__ __forceinline__ void unpack_row32(const uint32_t *w, float *v, const QuantParams &p) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        uint32_t u = w[j];
        if constexpr (RHT) u ^= p.sgn_pair[j];
        v[2 * j] = bf16lo(u);
        v[2 * j + 1] = bf16hi(u);
    }
    if constexpr (RHT) fwht32_scaled<RHT>(v, rht_norm<RHT>());
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void stg_v4(void *p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// ---------------------------------------------------------------------------
// 1D row blocks: one thread per 32-element block, grid-stride.
// ---------------------------------------------------------------------------
template <int RHT, bool SR, bool MMA>
__global__ void __launch_bounds__(256) quant_row_kernel(const QuantParams p) {
    pdl_wait();
    pdl_trigger();
    const int64_t nb = p.cols >> 5;
    const int64_t total = p.rows * nb;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= total) return;
    int64_t r = b / nb, kb = b - r * nb;
    const int64_t sr_ = stride / nb, sk_ = stride - sr_ * nb;
    for (; b < total; b += stride) {
        const uint16_t *src = p.x + r * p.ld_x + (kb << 5);
        uint32_t w[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 t = ldg_nc_v4(src + 8 * q);
            w[4 * q] = t.x; w[4 * q + 1] = t.y; w[4 * q + 2] = t.z; w[4 * q + 3] = t.w;
        }
        uint4 packed;
        const uint64_t g0 = (uint64_t)(r * p.cols + (kb << 5)) + p.elem_offset;
        uint32_t code;
        if constexpr (RHT) {
            float2 P[16];
            unpack_row32_pairs<RHT>(w, P, p);
            code = quantize32_pairs<SR>(P, packed, g0, p.seed_lo, p.seed_hi, p.scale_rule);
        } else {
            float v[32];
            unpack_row32<0>(w, v, p);
            code = quantize32<SR>(v, packed, g0, p.seed_lo, p.seed_hi, p.scale_rule);
        }
        stg_v4(p.codes + r * p.ld_codes + (kb << 4), packed);
        if constexpr (MMA) p.scales[mma_scale_off(r, kb, p.katoms)] = (uint8_t)code;
        else p.scales[r * p.ld_scales + kb] = (uint8_t)code;
        r += sr_;
        kb += sk_;
        if (kb >= nb) { kb -= nb; ++r; }
    }
}

// Tile of the column dequantizer: 256 rows x 64 columns of the output.
constexpr int COL_TR = 256, COL_TC = 64;

// 16-byte global -> shared copy that bypasses L1 (cp.async.cg).
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}

// Row and column of tile t in a grid of `cols` tile columns, for a
// persistent CTA's sequence t0, t0 + step, t0 + 2 step, ...: 32-bit divisions
// when the walk starts, then additions only.  (A 64-bit division per tile cost
// the 2D quantizer about 4.5 of its 13.9 instructions per element.)
struct TileStep {
    uint32_t step, dr, dc, cols;
    __device__ __forceinline__ TileStep(uint32_t step_, uint32_t cols_)
        : step(step_), dr(step_ / cols_), dc(step_ % cols_), cols(cols_) {}
};
struct TileWalk {
    uint32_t t, r, c;
    __device__ __forceinline__ TileWalk(uint32_t t0, uint32_t cols) : t(t0), r(t0 / cols), c(t0 % cols) {}
    __device__ __forceinline__ void next(const TileStep &st) {
        t += st.step;
        r += st.dr;
        c += st.dc;
        if (c >= st.cols) { c -= st.cols; ++r; }
    }
};


// ---------------------------------------------------------------------------
// Parameters of the column quantizer and of the dual (row + column) quantizer.
// ---------------------------------------------------------------------------
struct DualParams {
    const uint16_t *x;
    int64_t rows, cols, ld_x;
    uint8_t *rcodes, *rscales;             // row output: [rows, cols/2], scales for (rows x cols)
    int64_t ld_rcodes, ld_rscales, r_katoms;
    uint8_t *ccodes, *cscales;             // column output: [cols, rows/2], scales for (cols x rows)
    int64_t ld_ccodes, ld_cscales, c_katoms;
    uint32_t seed_lo, seed_hi;
    int scale_rule;                        // MXFP4_SCALE_* >> 4
    uint64_t r_offset, c_offset;           // SR stream index of each output's first element
    int64_t c_sr_ld;                       // row length of the column output's SR view (the whole tensor's rows)
    uint32_t tiles_c, tiles_r;             // column tiles, row tiles
    uint32_t strip;                        // column quantizer: tiles per strip (at most 8)
    uint32_t sgn_bit[32];                  // RHT sign of element i (mod the RHT size) as bit 31
};

// ---------------------------------------------------------------------------
// 1D-column quantizer (blocks of 32 along rows; output [cols, rows / 2]).  A
// CTA streams 256 x 64 bf16 tiles (32 KB, unpadded) through a three-deep
// cp.async ring.  Warp w owns row block w of a tile, lane l the column pair
// (2l, 2l + 1): each of its 32 shared loads is one bf16x2 word of a row (a
// warp reads one 128-byte row, conflict-free), and the two columns travel as
// the two lanes of packed fp32 pairs through the sign flip, the butterfly,
// the normalisation and the scaling, one f32x2 instruction per two elements.
// Every lane takes the same operations in the same order as the scalar
// reference, so the results are bit-identical.  Codes are staged per tile as
// 64 output rows of 128 bytes (16-byte pieces swizzled by column pair) and
// leave as 128-byte runs; scale bytes are staged per strip of
// vertically adjacent tiles and leave as 8 bytes per tile and output row in
// one run.
// ---------------------------------------------------------------------------
constexpr int CQ_TR = 256, CQ_TC = 64, CQ_STAGES = 3, CQ_MAX_STRIP = 8;
constexpr int CQ_TILE_BYTES = CQ_TR * CQ_TC * 2;                       // 32 KB of bf16
constexpr int CQ_OUT_BYTES = CQ_TC * (CQ_TR / 2);                      // 8 KB of codes
constexpr int CQ_SPITCH = 2 * CQ_MAX_STRIP + 1;                        // scale words per output row (+1: banks)
constexpr int CQ_SCALE_BYTES = CQ_TC * CQ_SPITCH * 4;                 // a strip's scale bytes
constexpr int CQ_SMEM = CQ_STAGES * CQ_TILE_BYTES + CQ_OUT_BYTES + CQ_SCALE_BYTES;

// Butterfly stages h = 1 .. D/2 over the 32 rows of a column pair (both
// lanes at once); D = 16 transforms the two 16-row halves separately.
template <int D>
__device__ __forceinline__ void fwht_col_pairs(float2 *P) {
#pragma unroll
    for (int h = 1; h < D; h <<= 1) {
#pragma unroll
        for (int m = 0; m < 32; ++m) {
            if ((m & h) == 0) {
                const float2 a = P[m], b = P[m + h];
                P[m] = add2(a, b);
                P[m + h] = sub2(a, b);
            }
        }
    }
}

// Codes of one column (lane HI of the pairs) of scaled values: four groups of
// eight rows, each one 32-bit word of nibbles.
template <bool SR, bool HI>
__device__ __forceinline__ uint4 encode_col_lane(const float2 *P, uint64_t g0, uint32_t k0, uint32_t k1) {
    const uint64_t blk = g0 >> 2;    // g0 % 4 == 0
    uint32_t q[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        float w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = HI ? P[8 * g + j].y : P[8 * g + j].x;
        if constexpr (SR) q[g] = e2m1x8_sr(w, blk + 2 * g, k0, k1);
        else q[g] = e2m1x8_rn(w);
    }
    return make_uint4(q[0], q[1], q[2], q[3]);
}

// One column-pair job: rows rin .. rin + 31 of output rows (columns) oc and
// oc + 1, lane word m at src[m * wstride] of a staged tile (bf16 of column oc
// in the low half).  The codes of each column (16 bytes) and its scale code;
// a NaN block (scale code 0xFF) gets zero codes.
template <int RHT, bool SR>
__device__ __forceinline__ void col_pair_job(const uint32_t *src, int wstride, const DualParams &p, int64_t oc,
                                             int64_t rin, uint4 &qlo, uint4 &qhi, uint32_t &slo, uint32_t &shi) {
    float2 P[32];                            // (column oc, column oc + 1) at row rin + m
#pragma unroll
    for (int m = 0; m < 32; ++m) {
        // bf16 -> fp32 with the RHT sign: adding 2^31 flips bit 31
        const uint32_t u = src[m * wstride];
        const uint32_t sg = RHT ? p.sgn_bit[m] : 0u;
        P[m] = make_float2(__uint_as_float(u * 65536u + sg), __uint_as_float((u & 0xFFFF0000u) ^ sg));
    }
    if constexpr (RHT != 0) {
        const float cn = rht_norm<RHT>();
        fwht_col_pairs<RHT>(P);
#pragma unroll
        for (int m = 0; m < 32; ++m) P[m] = mul2(P[m], make_float2(cn, cn));
    }
    float alo = 0.0f, ahi = 0.0f;
#pragma unroll
    for (int m = 0; m < 32; m += 2) {
        alo = amax_nan2(alo, P[m].x, P[m + 1].x);
        ahi = amax_nan2(ahi, P[m].y, P[m + 1].y);
    }
    slo = scale_code_rule(alo, p.scale_rule);
    shi = scale_code_rule(ahi, p.scale_rule);
    // a NaN block's lane is scaled by 1 and its codes replaced by zeros
    const float2 inv = make_float2(slo == 0xFFu ? 1.0f : inv_scale_from_code(slo),
                                   shi == 0xFFu ? 1.0f : inv_scale_from_code(shi));
    if (p.scale_rule == 2) {
#pragma unroll
        for (int m = 0; m < 32; ++m) P[m] = mul2(mul2(P[m], make_float2(0.75f, 0.75f)), inv);
    } else {
#pragma unroll
        for (int m = 0; m < 32; ++m) P[m] = mul2(P[m], inv);
    }
    const uint64_t g0 = (uint64_t)(oc * p.c_sr_ld + rin) + p.c_offset;
    qlo = encode_col_lane<SR, false>(P, g0, p.seed_lo, p.seed_hi);
    qhi = encode_col_lane<SR, true>(P, g0 + (uint64_t)p.c_sr_ld, p.seed_lo, p.seed_hi);
    if (slo == 0xFFu) qlo = make_uint4(0, 0, 0, 0);
    if (shi == 0xFFu) qhi = make_uint4(0, 0, 0, 0);
}

template <int RHT, bool SR, bool MMA>
__global__ void __launch_bounds__(256, 2) quant_col_kernel(const DualParams p, const uint32_t nstrips) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) uint8_t cq_smem[];
    uint8_t *ring = cq_smem;
    uint4 *tout = reinterpret_cast<uint4 *>(cq_smem + CQ_STAGES * CQ_TILE_BYTES);
    uint32_t *ssc = reinterpret_cast<uint32_t *>(cq_smem + CQ_STAGES * CQ_TILE_BYTES + CQ_OUT_BYTES);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t strip = p.strip;
    // The CTA's tiles in order: strips S = blockIdx.x + j * gridDim.x (row band
    // w.r, column band w.c of the strip grid), tile k of each of its len tiles
    // (row band w.r * strip + k).  A strip index past nstrips stays past it.
    struct Pos {
        TileWalk w;
        uint32_t k, len;
    };
    auto strip_len_of = [&](uint32_t band) -> uint32_t {
        const uint32_t t0 = band * strip;
        return t0 + strip <= p.tiles_r ? strip : (t0 < p.tiles_r ? p.tiles_r - t0 : strip);
    };
    const TileStep st(gridDim.x, p.tiles_c);
    auto advance = [&](Pos &q) {
        if (q.k + 1 < q.len) {
            ++q.k;
        } else {
            q.w.next(st);
            q.k = 0;
            q.len = strip_len_of(q.w.r);
        }
    };
    auto load = [&](const Pos &q, int buf) {
        if (q.w.t < nstrips) {
            const int64_t r0 = (int64_t)(q.w.r * strip + q.k) * CQ_TR, c0 = (int64_t)q.w.c * CQ_TC;
            const int ch = tid & 7, row = tid >> 3;          // rows row + 32 i, 16-byte chunk ch
            const int64_t gc = c0 + 8 * ch;
            const uint16_t *src = p.x + (r0 + row) * p.ld_x + gc;
            uint8_t *dst = ring + buf * CQ_TILE_BYTES + row * 128 + 16 * ch;
            if (r0 + CQ_TR <= p.rows && c0 + CQ_TC <= p.cols) {
#pragma unroll
                for (int i = 0; i < 8; ++i) cp_async16(dst + i * 32 * 128, src + (int64_t)i * 32 * p.ld_x);
            } else if (gc < p.cols) {                          // cols % 8 == 0: a chunk is whole or absent
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (r0 + row + 32 * i < p.rows) cp_async16(dst + i * 32 * 128, src + (int64_t)i * 32 * p.ld_x);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    Pos cur{TileWalk(blockIdx.x, p.tiles_c), 0u, 0u};
    cur.len = strip_len_of(cur.w.r);
    Pos n1 = cur;
    advance(n1);
    Pos n2 = n1;
    advance(n2);
    load(cur, 0);
    load(n1, 1);
    for (int it = 0; cur.w.t < nstrips; ++it) {
        load(n2, (it + 2) % CQ_STAGES);                      // two tiles in flight while this one is quantized
        asm volatile("cp.async.wait_group 2;" ::: "memory");
        __syncthreads();
        const uint32_t band = cur.w.r, k = cur.k;
        const int64_t r0 = (int64_t)(band * strip + k) * CQ_TR, c0 = (int64_t)cur.w.c * CQ_TC;
        const int64_t rin = r0 + 32 * warp, oc = c0 + 2 * lane;
        if (rin < p.rows && oc < p.cols) {
            const uint32_t *src =
                reinterpret_cast<const uint32_t *>(ring + (it % CQ_STAGES) * CQ_TILE_BYTES) + warp * 32 * 32 + lane;
            uint4 qlo, qhi;
            uint32_t slo, shi;
            col_pair_job<RHT, SR>(src, 32, p, oc, rin, qlo, qhi, slo, shi);
            const int c = 2 * lane, sw = warp ^ (lane & 7);
            tout[c * 8 + sw] = qlo;
            tout[(c + 1) * 8 + sw] = qhi;
            uint8_t *sb = reinterpret_cast<uint8_t *>(ssc);
            sb[4 * (c * CQ_SPITCH + 2 * k) + warp] = (uint8_t)slo;
            sb[4 * ((c + 1) * CQ_SPITCH + 2 * k) + warp] = (uint8_t)shi;
        }
        __syncthreads();                                     // tile read; codes and scales staged
        const uint32_t ntiles = cur.len;
        const bool last = k + 1 == ntiles;
        // codes: 64 output rows x 8 chunks of 16 bytes; 8 lanes write one row's 128 bytes
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
            const int row = (tid >> 3) + 32 * pass, ch = tid & 7;
            const int64_t orow = c0 + row, rb = r0 + 32 * ch;
            if (orow < p.cols && rb < p.rows)
                stg_v4(p.ccodes + orow * p.ld_ccodes + (rb >> 1), tout[row * 8 + (ch ^ ((row >> 1) & 7))]);
        }
        if (last) {                                          // the strip's scales: 8 K-blocks per tile and output row
            const int64_t kb0 = (int64_t)band * strip * 8, nkb = p.rows >> 5;
            const uint8_t *sb = reinterpret_cast<const uint8_t *>(ssc);
            if constexpr (MMA) {
                // 4-byte pieces (one MMA atom row slot each); consecutive
                // threads take consecutive rows, 16 bytes apart in an atom
                for (uint32_t idx = tid; idx < CQ_TC * 2u * ntiles; idx += 256) {
                    const uint32_t a = idx / CQ_TC, row = idx % CQ_TC;
                    const int64_t orow = c0 + row, kb = kb0 + 4 * a;
                    if (orow < p.cols && kb < nkb) {
                        uint8_t *dst = p.cscales + mma_scale_off(orow, kb, p.c_katoms);
                        const uint32_t w = ssc[row * CQ_SPITCH + a];
                        if (kb + 4 <= nkb) *reinterpret_cast<uint32_t *>(dst) = w;
                        else for (int j = 0; j < 4 && kb + j < nkb; ++j) dst[j] = (uint8_t)(w >> (8 * j));
                    }
                }
            } else if (((reinterpret_cast<uintptr_t>(p.cscales) | (uintptr_t)p.ld_cscales) & 3u) == 0) {
                // row-major, word-aligned rows: consecutive threads write
                // consecutive words of one output row
                const uint32_t nw = 2u * ntiles;
                for (uint32_t idx = tid; idx < CQ_TC * nw; idx += 256) {
                    const uint32_t row = idx / nw, a = idx - row * nw;
                    const int64_t orow = c0 + row, kb = kb0 + 4 * a;
                    if (orow < p.cols && kb < nkb) {
                        uint8_t *dst = p.cscales + orow * p.ld_cscales + kb;
                        const uint32_t w = ssc[row * CQ_SPITCH + a];
                        if (kb + 4 <= nkb) *reinterpret_cast<uint32_t *>(dst) = w;
                        else for (int j = 0; j < 4 && kb + j < nkb; ++j) dst[j] = (uint8_t)(w >> (8 * j));
                    }
                }
            } else {
                // row-major, any alignment: consecutive threads write
                // consecutive bytes of one output row
                const uint32_t nb = 8u * ntiles;
                for (uint32_t idx = tid; idx < CQ_TC * nb; idx += 256) {
                    const uint32_t row = idx / nb, j = idx - row * nb;
                    const int64_t orow = c0 + row, kb = kb0 + j;
                    if (orow < p.cols && kb < nkb) p.cscales[orow * p.ld_cscales + kb] = sb[4 * row * CQ_SPITCH + j];
                }
            }
        }
        cur = n1;
        n1 = n2;
        advance(n2);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Dual output: 1D-row blocks (no RHT) and 1D-column blocks (optional RHT along
// rows) of the same tensor from one read.  The recipe quantizes activations
// and gradients both ways (row blocks for fprop and dgrad, blocks along
// tokens for wgrad).  Under round-to-nearest (SR runs the kernel below) a CTA
// streams 128 x 64 bf16 tiles through a three-deep cp.async ring (rows padded
// to 144 bytes, which keeps both access patterns conflict-free), and its
// warps specialise:
//   warps 0-3, column jobs: warp w takes row block w, lane l the column pair
//     (2l, 2l + 1) as packed fp32 lanes, as in the column quantizer; the
//     codes are staged so that each output row leaves as 64 contiguous bytes;
//   warps 4-7, row jobs: thread r takes row r of the tile, both of its 32-
//     element blocks (64 bytes each from shared memory), 32 bytes of codes.
// The two halves carry about the same instruction count per tile.
// ---------------------------------------------------------------------------
constexpr int DQ_TR = 128, DQ_TC = 64, DQ_STAGES = 3;
constexpr int DQ_PITCH = DQ_TC * 2 + 16;                               // staged bytes per tile row
constexpr int DQ_TILE_BYTES = DQ_TR * DQ_PITCH;                        // 18 KB
constexpr int DQ_OUT_BYTES = DQ_TC * (DQ_TR / 2);                      // 4 KB of column codes
constexpr int DQ_SMEM = DQ_STAGES * DQ_TILE_BYTES + DQ_OUT_BYTES;

template <int CRHT, bool MMA>
__global__ void __launch_bounds__(256, 2) quant_dual_kernel(const DualParams p, const uint32_t ntiles) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) uint8_t dq_smem[];
    uint8_t *ring = dq_smem;
    uint4 *tout = reinterpret_cast<uint4 *>(dq_smem + DQ_STAGES * DQ_TILE_BYTES);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto load = [&](const TileWalk &w, int buf) {
        if (w.t < ntiles) {
            const int64_t r0 = (int64_t)w.r * DQ_TR, c0 = (int64_t)w.c * DQ_TC;
            const int ch = tid & 7, row = tid >> 3;            // rows row + 32 i, 16-byte chunk ch
            const int64_t gc = c0 + 8 * ch;
            const uint16_t *src = p.x + (r0 + row) * p.ld_x + gc;
            uint8_t *dst = ring + buf * DQ_TILE_BYTES + row * DQ_PITCH + 16 * ch;
            if (r0 + DQ_TR <= p.rows && c0 + DQ_TC <= p.cols) {
#pragma unroll
                for (int i = 0; i < 4; ++i) cp_async16(dst + i * 32 * DQ_PITCH, src + (int64_t)i * 32 * p.ld_x);
            } else if (gc < p.cols) {                            // cols % 32 == 0: a chunk is whole or absent
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (r0 + row + 32 * i < p.rows) cp_async16(dst + i * 32 * DQ_PITCH, src + (int64_t)i * 32 * p.ld_x);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    const TileStep st(gridDim.x, p.tiles_c);
    TileWalk cur(blockIdx.x, p.tiles_c), w1 = cur, w2 = cur;
    w1.next(st);
    w2.next(st);
    w2.next(st);
    load(cur, 0);
    load(w1, 1);
    for (int it = 0; cur.t < ntiles; ++it) {
        // two tiles in flight while this one is quantized; the buffer loaded
        // here was read in the previous iteration, before its barrier
        load(w2, (it + 2) % DQ_STAGES);
        asm volatile("cp.async.wait_group 2;" ::: "memory");
        __syncthreads();
        const int64_t r0 = (int64_t)cur.r * DQ_TR, c0 = (int64_t)cur.c * DQ_TC;
        const uint8_t *tile = ring + (it % DQ_STAGES) * DQ_TILE_BYTES;
        if (warp < 4) {                                          // column pair (2 lane, 2 lane + 1), row block warp
            const int64_t rin = r0 + 32 * warp, oc = c0 + 2 * lane;
            if (rin < p.rows && oc < p.cols) {
                const uint32_t *src = reinterpret_cast<const uint32_t *>(tile + 32 * warp * DQ_PITCH) + lane;
                uint4 qlo, qhi;
                uint32_t slo, shi;
                col_pair_job<CRHT, false>(src, DQ_PITCH / 4, p, oc, rin, qlo, qhi, slo, shi);
                const int c = 2 * lane, sw = warp ^ (lane & 3);
                tout[c * 4 + sw] = qlo;
                tout[(c + 1) * 4 + sw] = qhi;
                const int64_t kb = rin >> 5;
                if constexpr (MMA) {
                    p.cscales[mma_scale_off(oc, kb, p.c_katoms)] = (uint8_t)slo;
                    p.cscales[mma_scale_off(oc + 1, kb, p.c_katoms)] = (uint8_t)shi;
                } else {
                    p.cscales[oc * p.ld_cscales + kb] = (uint8_t)slo;
                    p.cscales[(oc + 1) * p.ld_cscales + kb] = (uint8_t)shi;
                }
            }
        } else {                                                 // row r, both 32-element blocks
            const int r = tid - 128;
            const int64_t orow = r0 + r;
            if (orow < p.rows) {
                const uint4 *s4 = reinterpret_cast<const uint4 *>(tile + r * DQ_PITCH);
#pragma unroll 1
                for (int b = 0; b < 2; ++b) {
                    const int64_t gc = c0 + 32 * b;
                    if (gc < p.cols) {
                        const uint4 u[4] = {s4[4 * b], s4[4 * b + 1], s4[4 * b + 2], s4[4 * b + 3]};
                        uint4 q;
                        const uint64_t g0 = (uint64_t)(orow * p.cols + gc) + p.r_offset;
                        const uint32_t sc = quantize32_bf16<false>(u, q, g0, p.seed_lo, p.seed_hi, p.scale_rule);
                        const int64_t kb = gc >> 5;
                        stg_v4(p.rcodes + orow * p.ld_rcodes + kb * 16, q);
                        if constexpr (MMA) p.rscales[mma_scale_off(orow, kb, p.r_katoms)] = (uint8_t)sc;
                        else p.rscales[orow * p.ld_rscales + kb] = (uint8_t)sc;
                    }
                }
            }
        }
        __syncthreads();                                         // tile read; column codes staged
        {   // column codes: 64 output rows x 4 chunks of 16 bytes, 4 lanes per row
            const int row = tid >> 2, ch = tid & 3;
            const int64_t orow = c0 + row, rb = r0 + 32 * ch;
            if (orow < p.cols && rb < p.rows)
                stg_v4(p.ccodes + orow * p.ld_ccodes + (rb >> 1), tout[row * 4 + (ch ^ ((row >> 1) & 3))]);
        }
        cur = w1;
        w1 = w2;
        w2.next(st);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// The dual quantizer under stochastic rounding, where Philox4x32-10 and the
// SR decision bound the kernel by integer issue rather than by HBM: more warps
// per SM matter more than wide jobs.  A CTA takes one 64 x 128 tile (rows
// padded by 16 bytes) and each thread does one column job, 32 rows of one
// column held as the pairs (v[m], v[m + 16]) of the packed butterfly, and one
// row job, 32 columns of one row; 80 registers, three CTAs per SM.
constexpr int DS_TR = 64, DS_TC = 128, DS_PITCH = DS_TC + 8;          // bf16 per staged row

template <int CRHT, bool MMA>
__global__ void __launch_bounds__(256, 3) quant_dual_sr_kernel(const DualParams p, const uint32_t ntiles) {
    pdl_wait();
    pdl_trigger();
    __shared__ __align__(16) uint16_t tin[2][DS_TR * DS_PITCH];
    __shared__ __align__(16) uint4 tout[DS_TC * 2];         // column codes: 128 output rows x 32 bytes
    const int tid = threadIdx.x;
    auto load = [&](uint32_t t, int buf) {
        const int64_t r0 = (int64_t)(t / p.tiles_c) * DS_TR, c0 = (int64_t)(t % p.tiles_c) * DS_TC;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int idx = tid + 256 * i, row = idx / (DS_TC / 8), ch = idx % (DS_TC / 8);
            const int64_t gr = r0 + row, gc = c0 + 8 * ch;
            if (gr < p.rows && gc < p.cols) cp_async16(tin[buf] + row * DS_PITCH + 8 * ch, p.x + gr * p.ld_x + gc);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    uint32_t t = blockIdx.x;
    if (t < ntiles) load(t, 0);
    for (int it = 0; t < ntiles; t += gridDim.x, ++it) {
        // the next tile's load is in flight while this one is quantized
        const int buf = it & 1;
        const uint32_t tn = t + gridDim.x;
        if (tn < ntiles) {
            load(tn, buf ^ 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const uint16_t *tile = tin[buf];
        const int64_t r0 = (int64_t)(t / p.tiles_c) * DS_TR, c0 = (int64_t)(t % p.tiles_c) * DS_TC;
        {                                                    // column c, rows 32b .. 32b + 31
            const int c = tid % DS_TC, b = tid / DS_TC;
            const int64_t orow = c0 + c, rin = r0 + 32 * b;
            if (orow < p.cols && rin < p.rows) {
                const uint16_t *col = tile + 32 * b * DS_PITCH + c;
                float2 P[16];                        // (v[m], v[m + 16]): packed two-lane arithmetic
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    // bf16 -> fp32 with the RHT sign: adding 2^31 flips bit 31
                    const uint32_t u0 = (uint32_t)col[m * DS_PITCH] * 65536u + (CRHT ? p.sgn_bit[m] : 0u);
                    const uint32_t u1 = (uint32_t)col[(m + 16) * DS_PITCH] * 65536u + (CRHT ? p.sgn_bit[m + 16] : 0u);
                    P[m] = make_float2(__uint_as_float(u0), __uint_as_float(u1));
                }
                if constexpr (CRHT) {
                    const float cn = rht_norm<CRHT>();
                    fwht_pairs<CRHT>(P);
#pragma unroll
                    for (int m = 0; m < 16; ++m) P[m] = mul2(P[m], make_float2(cn, cn));
                }
                uint4 q;
                const uint64_t g0 = (uint64_t)(orow * p.c_sr_ld + rin) + p.c_offset;
                const uint32_t sc = quantize32_pairs<true>(P, q, g0, p.seed_lo, p.seed_hi, p.scale_rule);
                tout[c * 2 + (b ^ ((c >> 2) & 1))] = q;
                const int64_t kb = rin >> 5;
                if constexpr (MMA) p.cscales[mma_scale_off(orow, kb, p.c_katoms)] = (uint8_t)sc;
                else p.cscales[orow * p.ld_cscales + kb] = (uint8_t)sc;
            }
        }
        {                                                    // row r, columns 32b .. 32b + 31
            const int r = tid % DS_TR, b = tid / DS_TR;
            const int64_t orow = r0 + r, gc = c0 + 32 * b;
            if (orow < p.rows && gc < p.cols) {
                const uint4 *s4 = reinterpret_cast<const uint4 *>(tile + r * DS_PITCH + 32 * b);
                const uint4 u[4] = {s4[0], s4[1], s4[2], s4[3]};
                uint4 q;
                const uint64_t g0 = (uint64_t)(orow * p.cols + gc) + p.r_offset;
                const uint32_t sc = quantize32_bf16<true>(u, q, g0, p.seed_lo, p.seed_hi, p.scale_rule);
                const int64_t kb = gc >> 5;
                stg_v4(p.rcodes + orow * p.ld_rcodes + kb * 16, q);
                if constexpr (MMA) p.rscales[mma_scale_off(orow, kb, p.r_katoms)] = (uint8_t)sc;
                else p.rscales[orow * p.ld_rscales + kb] = (uint8_t)sc;
            }
        }
        __syncthreads();
        {   // column codes: 128 output rows x 2 chunks of 16 bytes, one chunk per thread
            const int row = tid >> 1, ch = tid & 1;
            const int64_t orow = c0 + row, rin = r0 + 32 * ch;
            if (orow < p.cols && rin < p.rows)
                stg_v4(p.ccodes + orow * p.ld_ccodes + (rin >> 1), tout[row * 2 + (ch ^ ((row >> 2) & 1))]);
        }
        __syncthreads();                                     // the load after next overwrites this buffer
    }
}

// ---------------------------------------------------------------------------
// 2D 32x32 blocks.  A CTA streams tiles of 8 blocks through a double-buffered
// shared-memory ring (cp.async of whole tile rows, so the global reads are
// coalesced): 32 x 256 (one block row) without the transposed copy, 128 x 64
// (four block rows, two block columns) with it, so that each row of the
// transposed operand receives 64 contiguous bytes from one CTA.  Warp w owns
// one block, lane l its row l (64 bytes from shared memory; the row pitch is
// padded by 16 bytes, which keeps these reads conflict-free); amax is a warp
// max.  The transposed copy is built through a byte-transposed 512-byte
// shared-memory tile per warp.
// ---------------------------------------------------------------------------
template <bool TRANS>
struct Q2Tile {
    static constexpr int BR = TRANS ? 4 : 1;          // block rows per tile
    static constexpr int BC = 8 / BR;                 // block columns per tile
    static constexpr int ROWS = 32 * BR, COLS = 32 * BC;
    static constexpr int PITCH = COLS + 8;            // bf16 per smem row
    static constexpr int CHUNKS = COLS / 8;           // 16-byte chunks per row
};


template <int RHT, bool SR, bool MMA, bool TRANS>
__global__ void __launch_bounds__(256, SR ? 3 : (RHT != 0 || TRANS ? 5 : 4)) quant_2d_kernel(const QuantParams p) {
    pdl_wait();
    pdl_trigger();
    using T = Q2Tile<TRANS>;
    __shared__ __align__(16) uint16_t tin[2][T::ROWS * T::PITCH];
    __shared__ __align__(16) uint8_t tb[8][16][32];   // per warp: byte j of row r at [j][r]
    // round-to-nearest without the RHT or the transposed copy: the codes (32 rows
    // x 8 blocks of 16 bytes, block b of row r at b ^ (r & 7)), stored
    // row-contiguously during the next tile, after its first barrier
    constexpr bool STAGE = !TRANS && !SR && RHT == 0;
    __shared__ __align__(16) uint4 ocodes[STAGE ? 2 : 1][STAGE ? 32 * 8 : 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t nbr = p.rows >> 5, nbc = p.cols >> 5;
    auto flush = [&](const TileWalk &w, int ob) {
        if constexpr (STAGE) {
            const int row = tid >> 3, ch = tid & 7;
            const int64_t br = w.r, bc = (int64_t)w.c * T::BC + ch;
            if (br < nbr && bc < nbc)
                stg_v4(p.codes + ((br << 5) + row) * p.ld_codes + (bc << 4), ocodes[ob][row * 8 + (ch ^ (row & 7))]);
        }
    };
    const uint32_t tiles_c = (uint32_t)((nbc + T::BC - 1) / T::BC);
    const uint32_t ntiles = (uint32_t)((nbr + T::BR - 1) / T::BR) * tiles_c;   // the launcher checks it fits
    auto load = [&](const TileWalk &w, int buf) {
        // thread tid copies 16-byte chunk ch of rows row0 + RSTEP i
        constexpr int RSTEP = 256 / T::CHUNKS;
        static_assert(256 % T::CHUNKS == 0 && T::ROWS % RSTEP == 0, "tile copy shape");
        const int row0 = tid / T::CHUNKS, ch = tid % T::CHUNKS;
        const int64_t r0 = (int64_t)w.r * T::ROWS, c0 = (int64_t)w.c * T::COLS;
        const uint16_t *src = p.x + (r0 + row0) * p.ld_x + c0 + 8 * ch;
        uint16_t *dst = tin[buf] + row0 * T::PITCH + 8 * ch;
        if (r0 + T::ROWS <= p.rows && c0 + T::COLS <= p.cols) {
#pragma unroll
            for (int i = 0; i < T::ROWS / RSTEP; ++i)
                cp_async16(dst + i * RSTEP * T::PITCH, src + (int64_t)i * RSTEP * p.ld_x);
        } else if (c0 + 8 * ch < p.cols) {
#pragma unroll
            for (int i = 0; i < T::ROWS / RSTEP; ++i)
                if (r0 + row0 + i * RSTEP < p.rows)
                    cp_async16(dst + i * RSTEP * T::PITCH, src + (int64_t)i * RSTEP * p.ld_x);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    const TileStep st(gridDim.x, tiles_c);
    TileWalk cur(blockIdx.x, tiles_c), nxt = cur, prv = cur;
    nxt.next(st);
    if (cur.t < ntiles) load(cur, 0);
    int last = 0;
    for (int it = 0; cur.t < ntiles; ++it) {
        const int buf = it & 1;
        last = buf;
        if (nxt.t < ntiles) {
            load(nxt, buf ^ 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        if (it > 0) flush(prv, buf ^ 1);                 // the previous tile's codes
        const int wr = warp / T::BC, wc = warp % T::BC;   // this warp's block within the tile
        const int64_t br = (int64_t)cur.r * T::BR + wr;
        const int64_t bc = (int64_t)cur.c * T::BC + wc;
        if (br < nbr && bc < nbc) {
            const int64_t r = (br << 5) + lane, c0 = bc << 5;
            const uint4 *s4 = reinterpret_cast<const uint4 *>(tin[buf] + (32 * wr + lane) * T::PITCH + 32 * wc);
            uint32_t w[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 u = s4[q];
                w[4 * q] = u.x; w[4 * q + 1] = u.y; w[4 * q + 2] = u.z; w[4 * q + 3] = u.w;
            }
            // the block's amax is the warp max of the lanes' row maxima.  A
            // lane's maximum is +0, positive or the canonical NaN 0x7FFFFFFF,
            // so the unsigned maximum of the bit patterns is the NaN-
            // propagating float maximum, bit for bit, in one reduction
            auto warp_amax = [](float amax) {
                uint32_t r;
                asm("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(__float_as_uint(amax)));
                return __uint_as_float(r);
            };
            uint4 packed;
            uint32_t code;
            const uint64_t g0 = (uint64_t)(r * p.cols + c0) + p.elem_offset;
            if constexpr (RHT) {
                // the row stays in the packed butterfly's pairs through scaling and rounding
                float2 P[16];
                unpack_row32_pairs<RHT>(w, P, p);
                code = quantize32_pairs_amax<SR>(P, warp_amax(amax_pairs(P)), packed, g0, p.seed_lo, p.seed_hi,
                                                 p.scale_rule);
            } else {
                float v[32];
                unpack_row32<0>(w, v, p);
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 32; i += 2) amax = amax_nan2(amax, v[i], v[i + 1]);
                code = quantize_groups<SR>(
                    warp_amax(amax),
                    [&](int q, float *u) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) u[j] = v[8 * q + j];
                    },
                    packed, g0, p.seed_lo, p.seed_hi, p.scale_rule);
            }
            if constexpr (STAGE) ocodes[buf][lane * 8 + (wc ^ (lane & 7))] = packed;
            else stg_v4(p.codes + r * p.ld_codes + (c0 >> 1), packed);
            if constexpr (MMA) {
                p.scales[mma_scale_off(r, bc, p.katoms)] = (uint8_t)code;
            } else {
                if (lane == 0) p.scales[br * p.ld_scales + bc] = (uint8_t)code;
            }
            if constexpr (TRANS) {
                // byte-transpose through shared memory: tb[j][row] = byte j of row
                const uint32_t pw[4] = {packed.x, packed.y, packed.z, packed.w};
#pragma unroll
                for (int j = 0; j < 16; ++j) tb[warp][j][lane] = (uint8_t)(pw[j >> 2] >> (8 * (j & 3)));
                __syncwarp();
                // lane c gathers byte c/2 of every row and keeps nibble c&1
                const uint4 *rowp = reinterpret_cast<const uint4 *>(&tb[warp][lane >> 1][0]);
                const uint4 a = rowp[0], b2 = rowp[1];
                const uint32_t bw[8] = {a.x, a.y, a.z, a.w, b2.x, b2.y, b2.z, b2.w};
                const int sh = 4 * (lane & 1);
                uint32_t o[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    // words 2q, 2q+1 hold rows 8q..8q+7 (one byte each)
                    const uint32_t lo = (bw[2 * q] >> sh) & 0x0F0F0F0Fu;      // nibbles of rows 8q..8q+3
                    const uint32_t hi = (bw[2 * q + 1] >> sh) & 0x0F0F0F0Fu;  // rows 8q+4..8q+7
                    // pack row pairs: out byte k = nib(2k) | nib(2k+1) << 4
                    const uint32_t lo2 = (lo | (lo >> 4)) & 0x00FF00FFu;      // bytes: r0|r1, r2|r3
                    const uint32_t hi2 = (hi | (hi >> 4)) & 0x00FF00FFu;
                    o[q] = (lo2 & 0xFFu) | ((lo2 >> 8) & 0xFF00u) | ((hi2 & 0xFFu) << 16) | ((hi2 << 8) & 0xFF000000u);
                }
                __syncwarp();
                const int64_t ct = c0 + lane;       // row of the transposed operand
                stg_v4(p.codes_t + ct * p.ld_codes_t + (br << 4), make_uint4(o[0], o[1], o[2], o[3]));
                if (p.scales_t) {
                    if constexpr (MMA) {
                        p.scales_t[mma_scale_off(ct, br, p.katoms_t)] = (uint8_t)code;
                    } else {
                        if (lane == 0) p.scales_t[bc * p.ld_scales_t + br] = (uint8_t)code;
                    }
                }
            }
        }
        __syncthreads();                     // the load after next overwrites this buffer
        prv = cur;
        cur = nxt;
        nxt.next(st);
    }
    if (prv.t < ntiles) flush(prv, last);               // the last tile's codes
}

// ---------------------------------------------------------------------------
// Dequantize.
// ---------------------------------------------------------------------------
struct DequantParams {
    const uint8_t *codes;
    int64_t ld_codes;
    const uint8_t *scales;
    int64_t ld_scales, katoms;
    int64_t rows, cols;   // output shape
    void *out;
    int64_t ld_out;
    uint32_t sgn_pair[16];
    uint32_t sgn_bit[32];                  // RHT sign of element i (mod the RHT size) as bit 31
    uint32_t sgn_word[32];                 // the same sign at bits 15 and 31 (both halves of a bf16 pair)
};


__device__ __forceinline__ void decode32(const uint4 q, uint32_t scode, float *v) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    if (scode == 0xFFu) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(0x7FFFFFFFu);
        return;
    }
    const float X = scale_from_code(scode);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(e2m1_value((w[i >> 3] >> (4 * (i & 7))) & 0xFu), X);
}

// E2M1 decode by table lookup.  For a block with scale code sc < 0xFF every
// decoded value mag(c) * 2^(sc - 127) is exact in fp32 and has zero low 16
// bits: at most two significant bits, the smallest nonzero value 2^-128 is the
// subnormal 0x00200000, and products of 2^128 or more are Inf.  So its bf16
// pattern is exactly its fp32 high half, and the fp32 value is that half
// shifted up.  The eight magnitudes' half-words are computed once per block
// (eight exact products) and split into a table of low bytes and one of high
// bytes (two registers each); byte permutes look up four codes at a time and
// interleave the bytes into bf16 pairs; one multiply per pair moves the two
// sign bits (bit 3 of each nibble) to bits 15 and 31.
struct DecodeTable {
    uint32_t lo0, lo1, hi0, hi1;    // byte m of {lo1:lo0} / {hi1:hi0}: low / high byte of magnitude m's bf16
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ DecodeTable decode_table(uint32_t sc) {
    const float X = scale_from_code(sc);
    uint32_t h[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) h[m] = __float_as_uint(__fmul_rn(e2m1_value((uint32_t)m), X)) >> 16;
    const uint32_t p01 = prmt(h[0], h[1], 0x5140u), p23 = prmt(h[2], h[3], 0x5140u);
    const uint32_t p45 = prmt(h[4], h[5], 0x5140u), p67 = prmt(h[6], h[7], 0x5140u);
    DecodeTable t;
    t.lo0 = prmt(p01, p23, 0x5410u);
    t.hi0 = prmt(p01, p23, 0x7632u);
    t.lo1 = prmt(p45, p67, 0x5410u);
    t.hi1 = prmt(p45, p67, 0x7632u);
    return t;
}

// Four codes (the nibbles of the low 16 bits of g) -> two bf16 pairs.
__device__ __forceinline__ void decode4_bf16(const DecodeTable &t, uint32_t g, uint32_t &p01, uint32_t &p23) {
    const uint32_t sel = g & 0x7777u;
    const uint32_t lb = prmt(t.lo0, t.lo1, sel), hb = prmt(t.hi0, t.hi1, sel);
    p01 = prmt(lb, hb, 0x5140u) | (((g & 0x0088u) * 0x01001000u) & 0x80008000u);
    p23 = prmt(lb, hb, 0x7362u) | (((g & 0x8800u) * 0x00010010u) & 0x80008000u);
}

// 32 codes of one block -> 16 bf16 pairs (pair p = elements 2p, 2p + 1),
// exactly the nearest bf16 of the fp32 decode (which is exact); a NaN scale
// gives NaN pairs.
__device__ __forceinline__ void decode32_bf16(const uint4 q, uint32_t sc, uint32_t *pairs) {
    if (sc == 0xFFu) {
#pragma unroll
        for (int i = 0; i < 16; ++i) pairs[i] = 0x7FFF7FFFu;
        return;
    }
    const DecodeTable t = decode_table(sc);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        decode4_bf16(t, w[j], pairs[4 * j], pairs[4 * j + 1]);
        decode4_bf16(t, w[j] >> 16, pairs[4 * j + 2], pairs[4 * j + 3]);
    }
}

// The same as fp32 values (NaN scale: the quiet NaN 0x7FFFFFFF).
__device__ __forceinline__ void decode32_f32(const uint4 q, uint32_t sc, float *v) {
    uint32_t pr[16];
    decode32_bf16(q, sc, pr);
    if (sc == 0xFFu) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(0x7FFFFFFFu);
        return;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        v[2 * i] = __uint_as_float(pr[i] << 16);
        v[2 * i + 1] = __uint_as_float(pr[i] & 0xFFFF0000u);
    }
}

// One block decoded and inverse-transformed before the sign flip: v = c_d
// H_d (decode(code) 2^e) per d-segment.  For scale codes 27..246 (e = code -
// 127 in [-100, 119]) the butterfly runs on the unscaled magnitudes
// {0, 0.5, ..., 6}: every partial sum is a multiple of 0.5 below 2^8, exact in
// fp32, and so is its image under 2^e in the scaled butterfly (no overflow:
// 192 2^119 < FLT_MAX; below the normal range sums of multiples of 2^-149 are
// exact too).  The normalisation then multiplies by K = fp32(c_d 2^e), exact
// for these e, and RN(S K) equals the scaled path's RN(c_d (S 2^e)) because
// both round the same real number.  The decode table is the constant one of
// scale code 127, so the per-block table products disappear.  Other codes
// (tiny or huge scales, NaN) take the scaled path.
template <int RHT>
__device__ __forceinline__ void decode_inverse_fwht32(const uint4 q, uint32_t sc, float *v) {
    if (sc - 27u <= 219u) {
        decode32_f32(q, 127u, v);
        const float K = __uint_as_float(__float_as_uint(rht_norm<RHT>()) + ((sc - 127u) << 23));
        fwht32_scaled<RHT>(v, K);
    } else {
        decode32_f32(q, sc, v);
        fwht32_scaled<RHT>(v, rht_norm<RHT>());
    }
}

// Two blocks a and b of the unscaled domain at once, as f16 pairs P[i] =
// (a_i low, b_i high).  The decoded magnitudes {0, 0.5, ..., 6} and every
// partial sum of the butterfly (multiples of 0.5 below 2^8) are exact in f16
// as in fp32, so the packed f16 butterfly, taken in the same stage order
// and pairing as the fp32 one, gives the same values, zeros' signs included.
// The decode is the hardware E2M1 -> f16 conversion of bytes whose low
// nibble is a code of a and high nibble the code of b at the same index.
__device__ __forceinline__ void e2m1x2x4_f16x2(uint32_t w, uint32_t &h0, uint32_t &h1, uint32_t &h2, uint32_t &h3) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3) : "r"(w));
}
__device__ __forceinline__ uint32_t hadd2_rn(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t hsub2_rn(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ float2 f16x2_to_f32(uint32_t p) {
    float2 r;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tcvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
        : "=f"(r.x), "=f"(r.y) : "r"(p));
    return r;
}
template <int RHT>
__device__ __forceinline__ void decode_pair_fwht_f16(const uint4 qa, const uint4 qb, uint32_t *P) {
    const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w}, wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        // bytes (a_{8k+2m}, b_{8k+2m}) and (a_{8k+2m+1}, b_{8k+2m+1}), m = 0..3
        const uint32_t ev = (wa[k] & 0x0F0F0F0Fu) | ((wb[k] << 4) & 0xF0F0F0F0u);
        const uint32_t od = ((wa[k] >> 4) & 0x0F0F0F0Fu) | (wb[k] & 0xF0F0F0F0u);
        e2m1x2x4_f16x2(ev, P[8 * k], P[8 * k + 2], P[8 * k + 4], P[8 * k + 6]);
        e2m1x2x4_f16x2(od, P[8 * k + 1], P[8 * k + 3], P[8 * k + 5], P[8 * k + 7]);
    }
#pragma unroll
    for (int h = 1; h < RHT; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (!(i & h)) {
                const uint32_t x = P[i], y = P[i + h];
                P[i] = hadd2_rn(x, y);
                P[i + h] = hsub2_rn(x, y);
            }
        }
    }
}
// K = fp32(c_d 2^e) of a scale code in the unscaled-domain range 27..246.
template <int RHT>
__device__ __forceinline__ float unscaled_norm(uint32_t sc) {
    return __uint_as_float(__float_as_uint(rht_norm<RHT>()) + ((sc - 127u) << 23));
}
__device__ __forceinline__ bool unscaled_ok(uint32_t sc) { return sc - 27u <= 219u; }

template <int RHT>
__device__ __forceinline__ void inverse_rht32(float *v, const uint32_t *sgn_pair) {
    if constexpr (RHT) {
        fwht32_scaled<RHT>(v, rht_norm<RHT>());
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            v[2 * j] = __uint_as_float(__float_as_uint(v[2 * j]) ^ (sgn_pair[j] << 16));
            v[2 * j + 1] = __uint_as_float(__float_as_uint(v[2 * j + 1]) ^ (sgn_pair[j] & 0x80000000u));
        }
    }
}

// SMODE: 0 = row-major per row [rows, cols/32], 1 = row-major 2D tiles
// [rows/32, cols/32], 2 = MMA layout per row.
// One 32-value block decoded, inverse-transformed and rounded to 16 bf16
// pairs (pair j = elements 2j, 2j + 1); the RHT signs are applied to the
// rounded pairs (sgn_pair[j] holds them at bits 15 and 31), which equals
// flipping the fp32 values first since rounding to nearest is symmetric.
template <int RHT>
__device__ __forceinline__ void column_rht_bf16(const uint4 q, uint32_t sc, const uint32_t *sgn_pair,
                                                uint32_t *pairs) {
    float v[32];
    decode_inverse_fwht32<RHT>(q, sc, v);
#pragma unroll
    for (int j = 0; j < 16; ++j) pairs[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]) ^ sgn_pair[j];
}
template <int SMODE>
__device__ __forceinline__ uint32_t dequant_scale(const DequantParams &p, int64_t r, int64_t kb) {
    if constexpr (SMODE == 0) return p.scales[r * p.ld_scales + kb];
    else if constexpr (SMODE == 1) return p.scales[(r >> 5) * p.ld_scales + kb];
    else return p.scales[mma_scale_off(r, kb, p.katoms)];
}

// One block decoded (and inverse-transformed) and stored by its own lane.
template <int RHT, bool F32>
__device__ __forceinline__ void dequant_block_store(const DequantParams &p, int64_t r, int64_t kb, uint4 q,
                                                    uint32_t sc) {
    if constexpr (RHT == 0 && !F32) {
        // no transform, bf16 out: the looked-up pairs are the output
        uint32_t pr[16];
        decode32_bf16(q, sc, pr);
        uint16_t *dst = reinterpret_cast<uint16_t *>(p.out) + r * p.ld_out + (kb << 5);
#pragma unroll
        for (int i = 0; i < 4; ++i) stg_v4(dst + 8 * i, make_uint4(pr[4 * i], pr[4 * i + 1], pr[4 * i + 2], pr[4 * i + 3]));
        return;
    }
    float v[32];
    decode_inverse_fwht32<RHT>(q, sc, v);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        v[2 * j] = __uint_as_float(__float_as_uint(v[2 * j]) ^ (p.sgn_pair[j] << 16));
        v[2 * j + 1] = __uint_as_float(__float_as_uint(v[2 * j + 1]) ^ (p.sgn_pair[j] & 0x80000000u));
    }
    if constexpr (F32) {
        float *dst = reinterpret_cast<float *>(p.out) + r * p.ld_out + (kb << 5);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            stg_v4(dst + 4 * i, make_uint4(__float_as_uint(v[4 * i]), __float_as_uint(v[4 * i + 1]),
                                           __float_as_uint(v[4 * i + 2]), __float_as_uint(v[4 * i + 3])));
    } else {
        uint16_t *dst = reinterpret_cast<uint16_t *>(p.out) + r * p.ld_out + (kb << 5);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            stg_v4(dst + 8 * i, make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                                           pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7])));
    }
}

// A lane's two blocks with the inverse RHT, both scale codes in the
// unscaled-domain range: transformed together as f16 pairs; block 1's bf16
// output words (pair j = elements 2j, 2j + 1, RHT signs applied) go straight
// to the lane's slot, block 2's are returned in w2.
template <int RHT>
__device__ __forceinline__ void rht_pair_stage(uint4 q1, uint32_t s1, uint4 q2, uint32_t s2, const uint32_t *sgn_pair,
                                               uint4 *slot, int lane, uint32_t *w2) {
    uint32_t P[32];
    decode_pair_fwht_f16<RHT>(q1, q2, P);
    const float2 K2 = make_float2(unscaled_norm<RHT>(s1), unscaled_norm<RHT>(s2));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t a[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int j = 4 * i + m;
            const float2 f0 = mul2(f16x2_to_f32(P[2 * j]), K2), f1 = mul2(f16x2_to_f32(P[2 * j + 1]), K2);
            a[m] = pack_bf16x2(f0.x, f1.x) ^ sgn_pair[j];
            w2[j] = pack_bf16x2(f0.y, f1.y) ^ sgn_pair[j];
        }
        slot[4 * lane + (i ^ ((lane >> 1) & 3))] = make_uint4(a[0], a[1], a[2], a[3]);
    }
}

// A block's 16 bf16 output words into a lane's slot (layout as below).
__device__ __forceinline__ void stage_words_bf16(const uint32_t *w, uint4 *slot, int lane) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
        slot[4 * lane + (i ^ ((lane >> 1) & 3))] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

// One block's output words without a transform (16 bf16 pairs or 32 fp32)
// into a lane's slot of the warp's staging area: 16-byte unit q of lane l at
// unit 4l + (q ^ ((l >> 1) & 3)) (bf16; fp32: 8l + (q ^ (l & 7))), so that
// eight lanes' stores cover all 32 banks.
template <bool F32>
__device__ __forceinline__ void dequant_block_stage(uint4 q, uint32_t sc, uint4 *slot, int lane) {
    if constexpr (!F32) {
        uint32_t pr[16];                     // the looked-up pairs are the output
        decode32_bf16(q, sc, pr);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            slot[4 * lane + (i ^ ((lane >> 1) & 3))] = make_uint4(pr[4 * i], pr[4 * i + 1], pr[4 * i + 2], pr[4 * i + 3]);
    } else {
        float v[32];
        decode32_f32(q, sc, v);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            slot[8 * lane + (i ^ (lane & 7))] = make_uint4(__float_as_uint(v[4 * i]), __float_as_uint(v[4 * i + 1]),
                                                           __float_as_uint(v[4 * i + 2]), __float_as_uint(v[4 * i + 3]));
    }
}

// A warp's 32 staged blocks to global memory: in pass k lane l writes 16-byte
// unit 32k + l of the warp's run (block (32k + l) / U, unit (32k + l) % U, U
// units per block), so each store instruction covers 512 contiguous bytes
// where the blocks are contiguous.  `dst` is this lane's block's output
// address (null for no block); each unit takes its block's from that lane.
template <bool F32>
__device__ __forceinline__ void dequant_warp_store(const uint4 *slot, uint8_t *dst, int lane) {
    constexpr int U = F32 ? 8 : 4;
    __syncwarp();
#pragma unroll
    for (int k = 0; k < U; ++k) {
        const int c = 32 * k + lane, j = c / U, u = c % U;
        const uint64_t d = __shfl_sync(0xFFFFFFFFu, reinterpret_cast<uint64_t>(dst), j);
        if (d) {
            const int pos = F32 ? U * j + (u ^ (j & 7)) : U * j + (u ^ ((j >> 1) & 3));
            stg_v4(reinterpret_cast<uint8_t *>(d) + 16 * u, slot[pos]);
        }
    }
    __syncwarp();
}

// One 32-element block per thread and grid-stride step, two steps per loop
// iteration: both blocks' code and scale loads are issued before either is
// decoded, so each thread keeps two loads in flight.  Without the RHT a
// lane's block output (64 bytes bf16, 128 fp32) is staged in shared memory
// and the warp writes its 32 blocks with stores whose lanes cover consecutive
// 16-byte units: 16-byte stores at a 64-byte lane stride (each lane writing
// its own block) write half sectors per instruction, which held a 1:4
// read:write stream to 4.0 TB/s against 5.5 TB/s coalesced.
template <int RHT, bool F32, int SMODE>
__global__ void __launch_bounds__(256, RHT ? (F32 ? 3 : 2) : (F32 ? 2 : 4)) dequant_row_kernel(const DequantParams p) {
    pdl_wait();
    pdl_trigger();
    constexpr bool STAGED = RHT == 0 || !F32;
    __shared__ __align__(16) uint4 stage_all[STAGED ? 8 : 1][STAGED ? 32 * (F32 ? 8 : 4) : 1];
    const int lane = threadIdx.x & 31;
    uint4 *slot = stage_all[STAGED ? threadIdx.x >> 5 : 0];
    const int64_t nb = p.cols >> 5;
    const int64_t total = p.rows * nb;
    // (row, block) of the flat index b, stepped by the grid stride without a
    // division per iteration
    const int64_t b0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x, stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t dr = stride / nb, dk = stride - dr * nb;
    int64_t rr = b0 / nb, kk = b0 - rr * nb;
    auto step = [&](int64_t &r_, int64_t &k_) {
        r_ = rr;
        k_ = kk;
        rr += dr;
        kk += dk;
        if (kk >= nb) { kk -= nb; ++rr; }
    };
    auto out_at = [&](int64_t r_, int64_t k_) {
        return static_cast<uint8_t *>(p.out) + (r_ * p.ld_out + (k_ << 5)) * (F32 ? 4 : 2);
    };
    // the warp's lanes hold consecutive flat indices: it runs the loop as a
    // whole while any lane has a block
    const int64_t wb0 = b0 - lane;
    auto load_block = [&](bool has, int64_t r_, int64_t k_, uint4 &q, uint32_t &sc) {
        q = has ? ldg_nc_v4(p.codes + r_ * p.ld_codes + (k_ << 4)) : make_uint4(0, 0, 0, 0);
        sc = has ? dequant_scale<SMODE>(p, r_, k_) : 0u;
    };
    if constexpr (RHT != 0 && !F32) {
        // bf16 with the inverse RHT: both blocks transformed together, then
        // staged and stored like the blocks without it.  At two CTAs per SM
        // the next iteration's blocks are loaded before this one's are
        // processed, so each lane keeps four loads in flight.
        int64_t r1, k1, r2, k2;
        step(r1, k1);
        step(r2, k2);
        uint4 q1, q2;
        uint32_t s1, s2;
        load_block(b0 < total, r1, k1, q1, s1);
        load_block(b0 + stride < total, r2, k2, q2, s2);
        for (int64_t b = b0, wb = wb0; wb < total; b += 2 * stride, wb += 2 * stride) {
            const bool first = b < total, second = b + stride < total;
            int64_t nr1, nk1, nr2, nk2;
            step(nr1, nk1);
            step(nr2, nk2);
            uint4 nq1, nq2;
            uint32_t ns1, ns2;
            load_block(b + 2 * stride < total, nr1, nk1, nq1, ns1);
            load_block(b + 3 * stride < total, nr2, nk2, nq2, ns2);
            const bool pair = unscaled_ok(s1) && unscaled_ok(s2);
            uint32_t w2[16];
            if (pair) {
                rht_pair_stage<RHT>(q1, s1, q2, s2, p.sgn_pair, slot, lane, w2);
            } else {
                uint32_t w1[16];
                column_rht_bf16<RHT>(q1, s1, p.sgn_pair, w1);
                stage_words_bf16(w1, slot, lane);
            }
            dequant_warp_store<false>(slot, first ? out_at(r1, k1) : nullptr, lane);
            if (wb + stride < total) {
                if (!pair) column_rht_bf16<RHT>(q2, s2, p.sgn_pair, w2);
                stage_words_bf16(w2, slot, lane);
                dequant_warp_store<false>(slot, second ? out_at(r2, k2) : nullptr, lane);
            }
            r1 = nr1; k1 = nk1; r2 = nr2; k2 = nk2;
            q1 = nq1; q2 = nq2; s1 = ns1; s2 = ns2;
        }
    } else {
        for (int64_t b = b0, wb = wb0; wb < total; b += 2 * stride, wb += 2 * stride) {
            int64_t r1, k1, r2, k2;
            step(r1, k1);
            step(r2, k2);
            const bool first = b < total, second = b + stride < total;
            uint4 q1, q2;
            uint32_t s1, s2;
            load_block(first, r1, k1, q1, s1);
            load_block(second, r2, k2, q2, s2);
            if constexpr (RHT == 0) {
                if (first) dequant_block_stage<F32>(q1, s1, slot, lane);
                dequant_warp_store<F32>(slot, first ? out_at(r1, k1) : nullptr, lane);
                if (wb + stride < total) {
                    if (second) dequant_block_stage<F32>(q2, s2, slot, lane);
                    dequant_warp_store<F32>(slot, second ? out_at(r2, k2) : nullptr, lane);
                }
            } else {
                // fp32 with the inverse RHT: bound by its arithmetic, each
                // lane stores its own blocks
                if (first) dequant_block_store<RHT, F32>(p, r1, k1, q1, s1);
                if (second) dequant_block_store<RHT, F32>(p, r2, k2, q2, s2);
            }
        }
    }
}

// Transposed-view codes [cols, rows/2] back to out[rows, cols].  A tile is
// 64 code rows (= output columns) x 8 blocks (= 256 output rows): the codes
// are staged with coalesced 16-byte cp.async loads into a two-tile ring (three
// for bf16 with the RHT), the next tiles' loads in flight while this one is
// decoded (persistent grid).  Warp w decodes block w, lane l the output
// columns 2l and 2l+1 (bf16: both at once; fp32: one at a time, so that one
// 32-value block is live) and writes its 32 values per column down a per-warp
// 32-row shared tile, which the warp then writes to global memory with
// 16-byte stores, 128 (bf16) or 256 (fp32) contiguous bytes per row.  bf16
// with the RHT skips the tile: a lane's row word goes straight to its output
// row, 128 contiguous bytes per warp store.  The fp32 tile swaps word pairs of
// columns 32..63 so that the column writes of lanes l and l + 16 fall in
// different banks.
template <bool F32>
__host__ __device__ constexpr int dequant_col_row_bytes() { return COL_TC * (F32 ? 4 : 2); }
// bf16 output with the inverse RHT stores each row word directly (the
// transposing tile is only for the other outputs) and spends the shared
// memory saved on a three-tile code ring.
template <int RHT, bool F32>
__host__ __device__ constexpr bool dequant_col_direct() { return RHT != 0 && !F32; }
template <int RHT, bool F32>
__host__ __device__ constexpr int dequant_col_stages() { return dequant_col_direct<RHT, F32>() ? 3 : 2; }
template <int RHT, bool F32>
__host__ __device__ constexpr int dequant_col_smem() {
    return (int)sizeof(uint4) * dequant_col_stages<RHT, F32>() * COL_TC * 8 +
           (dequant_col_direct<RHT, F32>() ? 0 : 8 * 32 * dequant_col_row_bytes<F32>());
}

template <int RHT, bool F32, bool MMA>
__global__ void __launch_bounds__(256, (F32 || RHT) ? 2 : 4) dequant_col_kernel(const DequantParams p) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) uint8_t dyn_smem[];
    constexpr int ROWB = dequant_col_row_bytes<F32>();               // staged bytes per output row
    constexpr int CH = ROWB / 16;                                    // 16-byte chunks per row
    constexpr bool DIRECT = dequant_col_direct<RHT, F32>();
    constexpr int NST = dequant_col_stages<RHT, F32>();
    uint4 (*tin)[COL_TC][8] = reinterpret_cast<uint4 (*)[COL_TC][8]>(dyn_smem);   // NST x 8 KB of codes
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // chunk ch of staged code row `row` sits at ch ^ ((row >> 1) & 7): the
    // lanes of a warp read block `warp` of rows 2l, 2l + 1 (256 bytes apart),
    // which this spreads over all banks
    const int wsw = warp ^ (lane & 7);
    uint8_t *stage = dyn_smem + sizeof(uint4) * NST * COL_TC * 8 + warp * 32 * ROWB;   // unless DIRECT
    const uint32_t tiles_r = (uint32_t)((p.rows + COL_TR - 1) / COL_TR);
    const uint32_t tiles_c = (uint32_t)((p.cols + COL_TC - 1) / COL_TC);
    const uint32_t ntiles = tiles_r * tiles_c;                         // the launcher checks it fits
    auto load = [&](const TileWalk &w, int buf) {
        const int64_t r0 = (int64_t)w.r * COL_TR, c0 = (int64_t)w.c * COL_TC;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int row = (tid >> 3) + 32 * i, ch = tid & 7;
            const int64_t crow = c0 + row, rin = r0 + 32 * ch;
            if (crow < p.cols && rin < p.rows)
                cp_async16(&tin[buf][row][ch ^ ((row >> 1) & 7)], p.codes + crow * p.ld_codes + (rin >> 1));
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // the bf16 path's two scale bytes (columns 2l, 2l + 1 of row block w) of a
    // tile, loaded one tile ahead so that their latency hides behind a tile
    auto scale_pair = [&](const TileWalk &w, uint32_t &s0, uint32_t &s1) {
        s0 = s1 = 0xFFu;
        if (w.t < ntiles) {
            const int64_t rb = (int64_t)w.r * COL_TR + 32 * warp, oc = (int64_t)w.c * COL_TC + 2 * lane;
            if (rb < p.rows && oc < p.cols) {
                const int64_t kb = rb >> 5;
                s0 = MMA ? p.scales[mma_scale_off(oc, kb, p.katoms)] : p.scales[oc * p.ld_scales + kb];
                s1 = MMA ? p.scales[mma_scale_off(oc + 1, kb, p.katoms)] : p.scales[(oc + 1) * p.ld_scales + kb];
            }
        }
    };
    const TileStep st(gridDim.x, tiles_c);
    TileWalk cur(blockIdx.x, tiles_c), w1 = cur, w2 = cur;           // this tile, the next two
    w1.next(st);
    if (cur.t < ntiles) load(cur, 0);
    if constexpr (NST == 3) {
        w2 = w1;
        w2.next(st);
        load(w1, 1);                                                  // tiles past the end load nothing
    }
    uint32_t sa = 0xFFu, sb = 0xFFu;
    if constexpr (!F32) scale_pair(cur, sa, sb);
    for (int it = 0; cur.t < ntiles; ++it) {
        // NST - 1 tiles in flight while this one is decoded; the buffer
        // refilled here was read in an earlier iteration, before a barrier
        // every warp has passed
        const int buf = it % NST;
        uint32_t sa_n = 0xFFu, sb_n = 0xFFu;
        if constexpr (!F32) scale_pair(w1, sa_n, sb_n);
        if constexpr (NST == 3) {
            load(w2, (it + 2) % 3);
            asm volatile("cp.async.wait_group 2;" ::: "memory");
        } else if (w1.t < ntiles) {
            load(w1, buf ^ 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const int64_t r0 = (int64_t)cur.r * COL_TR, c0 = (int64_t)cur.c * COL_TC;
        const int64_t rb = r0 + 32 * warp;
        if (rb < p.rows) {
          const int64_t kb = rb >> 5;
          if constexpr (!F32) {
            // bf16 out: one 32-bit word (columns 2l, 2l + 1) per row, into
            // the staged tile, or with the RHT straight to the output row
            // (a warp's store then covers 128 contiguous bytes)
            const int64_t oc = c0 + 2 * lane;
            if (oc < p.cols) {                 // cols is even: oc + 1 < cols too
                uint32_t *w = DIRECT ? reinterpret_cast<uint32_t *>(static_cast<uint16_t *>(p.out) + rb * p.ld_out + oc)
                                     : reinterpret_cast<uint32_t *>(stage) + lane;
                const int64_t RW = DIRECT ? p.ld_out / 2 : ROWB / 4;   // 32-bit words between rows
                if constexpr (RHT == 0) {
                    // each column as 16 looked-up bf16 pairs along its rows
                    uint32_t pa[16], pb[16];
                    decode32_bf16(tin[buf][2 * lane][wsw], sa, pa);
                    decode32_bf16(tin[buf][2 * lane + 1][wsw], sb, pb);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        w[(2 * i) * RW] = prmt(pa[i], pb[i], 0x5410u);
                        w[(2 * i + 1) * RW] = prmt(pa[i], pb[i], 0x7632u);
                    }
                } else if (unscaled_ok(sa) && unscaled_ok(sb)) {
                    // both columns at once in the unscaled domain: row i of
                    // the pair is one f16 pair, then one fp32 pair scaled by
                    // (K_a, K_b), rounded to the bf16 pair of the staged word
                    uint32_t P[32];
                    decode_pair_fwht_f16<RHT>(tin[buf][2 * lane][wsw], tin[buf][2 * lane + 1][wsw], P);
                    const float2 K2 = make_float2(unscaled_norm<RHT>(sa), unscaled_norm<RHT>(sb));
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float2 f = mul2(f16x2_to_f32(P[i]), K2);
                        w[i * RW] = pack_bf16x2(f.x, f.y) ^ p.sgn_word[i];
                    }
                } else {
                    // each column decoded, transformed, rounded and
                    // sign-flipped as 16 bf16 pairs along its rows
                    uint32_t pa[16], pb[16];
                    column_rht_bf16<RHT>(tin[buf][2 * lane][wsw], sa, p.sgn_pair, pa);
                    column_rht_bf16<RHT>(tin[buf][2 * lane + 1][wsw], sb, p.sgn_pair, pb);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        w[(2 * i) * RW] = prmt(pa[i], pb[i], 0x5410u);
                        w[(2 * i + 1) * RW] = prmt(pa[i], pb[i], 0x7632u);
                    }
                }
            }
          } else {
            // fp32 out: one column at a time, one 32-value block live
#pragma unroll 1
            for (int j = 0; j < 2; ++j) {
                const int c = 2 * lane + j;
                const int64_t oc = c0 + c;
                if (oc < p.cols) {
                    const uint32_t sc = MMA ? p.scales[mma_scale_off(oc, kb, p.katoms)] : p.scales[oc * p.ld_scales + kb];
                    float v[32];
                    if constexpr (RHT) {
                        decode_inverse_fwht32<RHT>(tin[buf][c][wsw], sc, v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(__float_as_uint(v[i]) ^ p.sgn_bit[i % RHT]);
                    } else {
                        decode32_f32(tin[buf][c][wsw], sc, v);
                    }
                    const int wpos = c ^ ((c >> 5) & 1);                // bank-spreading word swap
                    uint32_t *col = reinterpret_cast<uint32_t *>(stage) + wpos;
#pragma unroll
                    for (int i = 0; i < 32; ++i) col[i * (ROWB / 4)] = __float_as_uint(v[i]);
                }
            }
          }
          if constexpr (!DIRECT) {
            __syncwarp();
            // 32 rows of ROWB bytes: lane-contiguous 16-byte chunks of each row
#pragma unroll
            for (int idx = lane; idx < 32 * CH; idx += 32) {
                const int row = idx / CH, ch = idx - row * CH;
                const int64_t col0 = c0 + ch * (16 / (F32 ? 4 : 2));
                if (col0 < p.cols) {
                    uint4 w = *reinterpret_cast<const uint4 *>(stage + row * ROWB + ch * 16);
                    if constexpr (F32) {
                        if (ch >= CH / 2) w = make_uint4(w.y, w.x, w.w, w.z);   // undo the word swap
                    }
                    uint8_t *dst = static_cast<uint8_t *>(p.out) + ((rb + row) * p.ld_out + col0) * (F32 ? 4 : 2);
                    stg_v4(dst, w);
                }
            }
            __syncwarp();
          }
        }
        __syncthreads();
        sa = sa_n;
        sb = sb_n;
        cur = w1;
        if constexpr (NST == 3) {
            w1 = w2;
            w2.next(st);
        } else {
            w1.next(st);
        }
    }
    if constexpr (NST == 3) asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Host-side launchers (called by the C ABI after validation).
// ---------------------------------------------------------------------------
static int g_num_sms = 0;

static int num_sms() {
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (g_num_sms <= 0) g_num_sms = 148;
    }
    return g_num_sms;
}

// Resident CTAs per SM of a kernel (persistent grids are SMs x this).
// Cached per kernel; the value depends only on the kernel and block size.
static int resident_ctas(const void *kern, int threads, size_t dyn_smem = 0) {
    static std::mutex mu;
    static std::map<const void *, int> cache;
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(kern);
    if (it != cache.end()) return it->second;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, dyn_smem) != cudaSuccess || occ <= 0)
        occ = 1;
    cache[kern] = occ;
    return occ;
}

// Dynamic shared memory above the 48 KB default: the opt-in, once per kernel
// and device.
static cudaError_t allow_dyn_smem(const void *kern, int bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, bool> done;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({kern, dev})) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[{kern, dev}] = true;
    return e;
}

static void fill_signs(uint32_t mask, int rht, uint32_t *pair, uint32_t *bit) {
    for (int j = 0; j < 16; ++j) {
        const uint32_t e0 = (uint32_t)(2 * j) % (uint32_t)(rht ? rht : 32);
        const uint32_t e1 = (uint32_t)(2 * j + 1) % (uint32_t)(rht ? rht : 32);
        const uint32_t s0 = rht ? (mask >> e0) & 1u : 0u;
        const uint32_t s1 = rht ? (mask >> e1) & 1u : 0u;
        pair[j] = (s0 << 15) | (s1 << 31);
    }
    for (int i = 0; i < 32; ++i) {
        const uint32_t s = rht ? (mask >> (i % rht)) & 1u : 0u;
        bit[i] = s ? 0x80000000u : 0u;
    }
}

// Grid of the grid-stride row kernels: about 14 items per thread, between 4
// and 32 CTAs per SM.  Small tensors then run as resident CTAs that each loop
// several times (a 64 MiB row quantize: 0.63 -> 0.70 of HBM against one item
// per thread), large ones oversubscribed (1 GiB: 0.96 against 0.88 with 4
// CTAs per SM).
static int64_t grid_for(int64_t items, int threads) {
    const int64_t g = (items + threads - 1) / threads;
    const int64_t lo = (int64_t)num_sms() * 4, hi = (int64_t)num_sms() * 32;
    int64_t want = (items + (int64_t)threads * 14 - 1) / ((int64_t)threads * 14);
    want = want < lo ? lo : (want > hi ? hi : want);
    const int64_t grid = g < want ? g : want;
    return grid < 1 ? 1 : grid;
}

template <int RHT, bool SR, bool MMA>
static cudaError_t launch_col_dual(const QuantParams &q, cudaStream_t s);

template <int RHT, bool SR, bool MMA>
static cudaError_t launch_quant_t(int layout, bool trans, const QuantParams &p, cudaStream_t s) {
    if (layout == MXFP4_LAYOUT_1D_ROW) {
        return launch_pdl(quant_row_kernel<RHT, SR, MMA>, dim3((unsigned)grid_for(p.rows * (p.cols / 32), 256)), dim3(256), 0, s, p);
    } else if (layout == MXFP4_LAYOUT_1D_COL) {
        return launch_col_dual<RHT, SR, MMA>(p, s);      // the column quantizer
    } else {
        const int br = trans ? Q2Tile<true>::BR : Q2Tile<false>::BR;
        const int64_t tiles = ((p.rows / 32 + br - 1) / br) * ((p.cols / 32 + 8 / br - 1) / (8 / br));
        if (tiles > 0xFFFFFFFFll - 0x7FFFFFFFll) return cudaErrorInvalidValue;   // tile index fits 32 bits
        auto kern = trans ? quant_2d_kernel<RHT, SR, MMA, true> : quant_2d_kernel<RHT, SR, MMA, false>;
        // persistent for RNE (memory-bound), one CTA per tile for SR (ALU-bound)
        int64_t cap = SR ? 0x7FFFFFFFll
                         : (int64_t)num_sms() * resident_ctas(reinterpret_cast<const void *>(kern), 256);
        if (tiles < 4 * cap) cap = tiles;                   // small tensors: one CTA per tile
        return launch_pdl(kern, dim3((unsigned)(tiles < cap ? tiles : cap)), dim3(256), 0, s, p);
    }
    return cudaGetLastError();
}

template <int RHT, bool SR>
static cudaError_t launch_quant_r(int layout, bool trans, bool mma, const QuantParams &p, cudaStream_t s) {
    return mma ? launch_quant_t<RHT, SR, true>(layout, trans, p, s) : launch_quant_t<RHT, SR, false>(layout, trans, p, s);
}

template <int RHT>
static cudaError_t launch_quant_s(int layout, bool trans, bool mma, bool sr, const QuantParams &p, cudaStream_t s) {
    return sr ? launch_quant_r<RHT, true>(layout, trans, mma, p, s) : launch_quant_r<RHT, false>(layout, trans, mma, p, s);
}

cudaError_t launch_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int layout, int rht,
                            int rounding, uint64_t seed, uint64_t elem_offset, uint8_t *codes, int64_t ld_codes,
                            uint8_t *scales, int64_t ld_scales, int scale_layout, uint8_t *codes_t,
                            int64_t ld_codes_t, uint8_t *scales_t, int64_t ld_scales_t, cudaStream_t s) {
    QuantParams p{};
    p.x = static_cast<const uint16_t *>(x);
    p.rows = rows; p.cols = cols; p.ld_x = ld_x;
    p.codes = codes; p.ld_codes = ld_codes;
    p.scales = scales; p.ld_scales = ld_scales;
    p.codes_t = codes_t; p.ld_codes_t = ld_codes_t;
    p.scales_t = scales_t; p.ld_scales_t = ld_scales_t;
    const int64_t k_out = layout == MXFP4_LAYOUT_1D_COL ? rows : cols;
    p.katoms = mma_katoms(k_out);
    p.katoms_t = mma_katoms(rows);
    p.seed_lo = (uint32_t)seed; p.seed_hi = (uint32_t)(seed >> 32);
    p.elem_offset = elem_offset;
    fill_signs(rht ? rht_sign_mask_hd(seed) : 0u, rht, p.sgn_pair, p.sgn_bit);
    const bool mma = scale_layout == MXFP4_SCALES_MMA;
    const bool sr = (rounding & 0x0F) == MXFP4_ROUND_SR;
    p.scale_rule = (rounding >> 4) & 3;
    const bool trans = codes_t != nullptr;
    switch (rht) {
        case 0: return launch_quant_s<0>(layout, trans, mma, sr, p, s);
        case 16: return launch_quant_s<16>(layout, trans, mma, sr, p, s);
        default: return launch_quant_s<32>(layout, trans, mma, sr, p, s);
    }
}

// Tiles per strip of the column-only RNE quantizer: the L in {1, 2, 4, 8}
// that minimises (strips of the busiest CTA) x L x (time per tile at L), over
// the L that still fill the persistent grid.  Time per tile relative to L = 1,
// measured on B200 with a 186,400 x 2880 bf16 tensor: 0.88 (L = 2), 0.815
// (4), 0.805 (8).
static uint32_t strip_len(uint64_t tiles_r, uint64_t tiles_c, uint64_t grid) {
    static const uint32_t cost[4] = {1000, 880, 815, 805};
    uint32_t best = 1;
    uint64_t best_t = ((tiles_r * tiles_c + grid - 1) / grid) * cost[0];
    for (int i = 1; i < 4; ++i) {
        const uint64_t L = 1ull << i, strips = (tiles_r + L - 1) / L * tiles_c;
        if (strips < grid) break;
        const uint64_t t = (strips + grid - 1) / grid * L * cost[i];
        if (t < best_t) { best_t = t; best = (uint32_t)L; }
    }
    return best;
}

// Both outputs under SR: one CTA per 64 x 128 tile (the hardware scheduler
// balances the tail of an issue-bound kernel).
template <int CRHT, bool MMA>
static cudaError_t launch_dual_sr(DualParams p, cudaStream_t s) {
    p.tiles_c = (uint32_t)((p.cols + DS_TC - 1) / DS_TC);
    const uint64_t tiles = (uint64_t)((p.rows + DS_TR - 1) / DS_TR) * p.tiles_c;
    if (tiles > 0x7FFFFFFFull) return cudaErrorInvalidValue;
    return launch_pdl(quant_dual_sr_kernel<CRHT, MMA>, dim3((unsigned)tiles), dim3(256), 0, s, p, (uint32_t)tiles);
}

// Both outputs: under RNE the dual quantizer, persistent at full occupancy.
template <int CRHT, bool SR, bool MMA>
static cudaError_t launch_dual_t(DualParams p, cudaStream_t s) {
    if constexpr (SR) {
        return launch_dual_sr<CRHT, MMA>(p, s);
    } else {
        p.tiles_c = (uint32_t)((p.cols + DQ_TC - 1) / DQ_TC);
        const uint64_t tiles_r = (uint64_t)((p.rows + DQ_TR - 1) / DQ_TR);
        const uint64_t tiles = tiles_r * p.tiles_c;
        if (tiles > 0xFFFFFFFFull - 0x7FFFFFFFull) return cudaErrorInvalidValue;   // tile index fits 32 bits
        p.tiles_r = (uint32_t)tiles_r;
        auto kern = quant_dual_kernel<CRHT, MMA>;
        const cudaError_t ea = allow_dyn_smem(reinterpret_cast<const void *>(kern), DQ_SMEM);
        if (ea != cudaSuccess) return ea;
        uint64_t cap =
            (uint64_t)num_sms() * (uint64_t)resident_ctas(reinterpret_cast<const void *>(kern), 256, DQ_SMEM);
        if (tiles < 4 * cap) cap = tiles;                   // small tensors: one CTA per tile
        return launch_pdl(kern, dim3((unsigned)(tiles < cap ? tiles : cap)), dim3(256), (size_t)DQ_SMEM, s, p,
                          (uint32_t)tiles);
    }
}

// Column output only: the column quantizer on 256 x 64 tiles, persistent at
// full occupancy (two CTAs per SM), strips as long as the grid stays full.
template <int RHT, bool SR, bool MMA>
static cudaError_t launch_col_t(DualParams p, cudaStream_t s) {
    p.tiles_c = (uint32_t)((p.cols + CQ_TC - 1) / CQ_TC);
    const uint64_t tiles_r = (uint64_t)((p.rows + CQ_TR - 1) / CQ_TR);
    if (tiles_r * p.tiles_c > 0xFFFFFFFFull - 0x7FFFFFFFull) return cudaErrorInvalidValue;
    p.tiles_r = (uint32_t)tiles_r;
    auto kern = quant_col_kernel<RHT, SR, MMA>;
    const cudaError_t ea = allow_dyn_smem(reinterpret_cast<const void *>(kern), CQ_SMEM);
    if (ea != cudaSuccess) return ea;
    const uint64_t cap =
        (uint64_t)num_sms() * (uint64_t)resident_ctas(reinterpret_cast<const void *>(kern), 256, CQ_SMEM);
    p.strip = tiles_r * p.tiles_c > 0 ? strip_len(tiles_r, p.tiles_c, cap) : 1u;
    if (p.strip > 4) p.strip = 4;
    const uint64_t strips = (tiles_r + p.strip - 1) / p.strip * p.tiles_c;
    return launch_pdl(kern, dim3((unsigned)(strips < cap ? strips : cap)), dim3(256), (size_t)CQ_SMEM, s, p,
                      (uint32_t)strips);
}

// 1D-column quantization through the column quantizer.
template <int RHT, bool SR, bool MMA>
static cudaError_t launch_col_dual(const QuantParams &q, cudaStream_t s) {
    DualParams p{};
    p.x = q.x;
    p.rows = q.rows; p.cols = q.cols; p.ld_x = q.ld_x;
    p.ccodes = q.codes; p.ld_ccodes = q.ld_codes;
    p.cscales = q.scales; p.ld_cscales = q.ld_scales; p.c_katoms = q.katoms;
    p.seed_lo = q.seed_lo; p.seed_hi = q.seed_hi;
    p.scale_rule = q.scale_rule;
    p.c_offset = q.elem_offset;
    p.c_sr_ld = q.rows;
    for (int i = 0; i < 32; ++i) p.sgn_bit[i] = q.sgn_bit[i];
    return launch_col_t<RHT, SR, MMA>(p, s);
}

template <int CRHT, bool SR, bool MMA>
static cudaError_t launch_dual_o(bool do_row, bool do_col, const DualParams &p, cudaStream_t s) {
    if (do_row && do_col) return launch_dual_t<CRHT, SR, MMA>(p, s);
    if (do_col) return launch_col_t<CRHT, SR, MMA>(p, s);
    // row output only: the row quantizer (no RHT) with the row output's offset
    QuantParams q{};
    q.x = p.x;
    q.rows = p.rows; q.cols = p.cols; q.ld_x = p.ld_x;
    q.codes = p.rcodes; q.ld_codes = p.ld_rcodes;
    q.scales = p.rscales; q.ld_scales = p.ld_rscales; q.katoms = p.r_katoms;
    q.seed_lo = p.seed_lo; q.seed_hi = p.seed_hi;
    q.scale_rule = p.scale_rule;
    q.elem_offset = p.r_offset;
    return launch_pdl(quant_row_kernel<0, SR, MMA>, dim3((unsigned)grid_for(q.rows * (q.cols / 32), 256)), dim3(256),
                      0, s, q);
}

template <int CRHT>
static cudaError_t launch_dual_r(bool sr, bool mma, bool do_row, bool do_col, const DualParams &p, cudaStream_t s) {
    if (sr) return mma ? launch_dual_o<CRHT, true, true>(do_row, do_col, p, s) : launch_dual_o<CRHT, true, false>(do_row, do_col, p, s);
    return mma ? launch_dual_o<CRHT, false, true>(do_row, do_col, p, s) : launch_dual_o<CRHT, false, false>(do_row, do_col, p, s);
}

cudaError_t launch_quantize_dual(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int col_rht, int rounding,
                                 uint64_t seed, uint64_t row_offset, uint64_t col_offset, uint8_t *rcodes,
                                 int64_t ld_rcodes, uint8_t *rscales, int64_t ld_rscales, uint8_t *ccodes,
                                 int64_t ld_ccodes, uint8_t *cscales, int64_t ld_cscales, int scale_layout,
                                 int64_t col_sr_ld, cudaStream_t s) {
    DualParams p{};
    p.x = static_cast<const uint16_t *>(x);
    p.rows = rows; p.cols = cols; p.ld_x = ld_x;
    p.rcodes = rcodes; p.rscales = rscales; p.ld_rcodes = ld_rcodes; p.ld_rscales = ld_rscales;
    p.r_katoms = mma_katoms(cols);
    p.ccodes = ccodes; p.cscales = cscales; p.ld_ccodes = ld_ccodes; p.ld_cscales = ld_cscales;
    p.c_katoms = mma_katoms(rows);
    p.seed_lo = (uint32_t)seed; p.seed_hi = (uint32_t)(seed >> 32);
    p.r_offset = row_offset; p.c_offset = col_offset;
    p.c_sr_ld = col_sr_ld > 0 ? col_sr_ld : rows;
    uint32_t pair_unused[16];
    fill_signs(col_rht ? rht_sign_mask_hd(seed) : 0u, col_rht, pair_unused, p.sgn_bit);
    const bool sr = (rounding & 0x0F) == MXFP4_ROUND_SR, mma = scale_layout == MXFP4_SCALES_MMA;
    p.scale_rule = (rounding >> 4) & 3;
    const bool do_row = rcodes != nullptr, do_col = ccodes != nullptr;
    switch (col_rht) {
        case 0: return launch_dual_r<0>(sr, mma, do_row, do_col, p, s);
        case 16: return launch_dual_r<16>(sr, mma, do_row, do_col, p, s);
        default: return launch_dual_r<32>(sr, mma, do_row, do_col, p, s);
    }
}

template <int RHT, bool F32>
static cudaError_t launch_dequant_t(int layout, int smode, const DequantParams &p, cudaStream_t s) {
    if (layout == MXFP4_LAYOUT_1D_COL) {
        // persistent at full occupancy: each CTA keeps its next tile's load in flight
        const int64_t tiles = ((p.rows + COL_TR - 1) / COL_TR) * ((p.cols + COL_TC - 1) / COL_TC);
        if (tiles > 0xFFFFFFFFll - 0x7FFFFFFFll) return cudaErrorInvalidValue;   // tile index fits 32 bits
        auto kern = smode == 2 ? dequant_col_kernel<RHT, F32, true> : dequant_col_kernel<RHT, F32, false>;
        constexpr int smem = dequant_col_smem<RHT, F32>();
        const cudaError_t ea = allow_dyn_smem(reinterpret_cast<const void *>(kern), smem);
        if (ea != cudaSuccess) return ea;
        const int64_t cap = (int64_t)num_sms() * resident_ctas(reinterpret_cast<const void *>(kern), 256, smem);
        const unsigned g = (unsigned)(tiles < cap ? tiles : cap);
        return launch_pdl(kern, dim3(g), dim3(256), (size_t)smem, s, p);
    } else {
        auto kern = smode == 0 ? dequant_row_kernel<RHT, F32, 0>
                               : (smode == 1 ? dequant_row_kernel<RHT, F32, 1> : dequant_row_kernel<RHT, F32, 2>);
        const int64_t items = p.rows * (p.cols / 32);
        int64_t g = grid_for(items, 256);
        if constexpr (RHT != 0 && !F32) {
            // the software-pipelined loop: one wave of resident CTAs, each
            // carrying its prefetch across all of its iterations
            const int64_t cap = (int64_t)num_sms() * resident_ctas(reinterpret_cast<const void *>(kern), 256, 0);
            const int64_t need = (items + 255) / 256;
            g = need < cap ? need : cap;
        }
        return launch_pdl(kern, dim3((unsigned)(g < 1 ? 1 : g)), dim3(256), 0, s, p);
    }
    return cudaGetLastError();
}

template <int RHT>
static cudaError_t launch_dequant_r(int layout, int smode, bool f32, const DequantParams &p, cudaStream_t s) {
    return f32 ? launch_dequant_t<RHT, true>(layout, smode, p, s) : launch_dequant_t<RHT, false>(layout, smode, p, s);
}

cudaError_t launch_dequantize(const uint8_t *codes, int64_t ld_codes, const uint8_t *scales, int64_t ld_scales,
                              int scale_layout, int64_t rows, int64_t cols, int layout, int rht, uint64_t seed,
                              void *out, int64_t ld_out, int out_dtype, cudaStream_t s) {
    DequantParams p{};
    p.codes = codes; p.ld_codes = ld_codes;
    p.scales = scales; p.ld_scales = ld_scales;
    p.rows = rows; p.cols = cols; p.out = out; p.ld_out = ld_out;
    p.katoms = mma_katoms(layout == MXFP4_LAYOUT_1D_COL ? rows : cols);
    fill_signs(rht ? rht_sign_mask_hd(seed) : 0u, rht, p.sgn_pair, p.sgn_bit);
    for (int i = 0; i < 32; ++i) p.sgn_word[i] = p.sgn_bit[i] | (p.sgn_bit[i] >> 16);
    const int smode = scale_layout == MXFP4_SCALES_MMA ? 2 : (layout == MXFP4_LAYOUT_2D ? 1 : 0);
    const bool f32 = out_dtype == MXFP4_OUT_F32;
    switch (rht) {
        case 0: return launch_dequant_r<0>(layout, smode, f32, p, s);
        case 16: return launch_dequant_r<16>(layout, smode, f32, p, s);
        default: return launch_dequant_r<32>(layout, smode, f32, p, s);
    }
}

}  // namespace mxfp4
