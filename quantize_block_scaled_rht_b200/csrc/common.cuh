// common.cuh -- device helpers shared by the MXFP4 kernels (sm_100a).
//
// Number format: "MXFP4" (aiwiki.ai), "Format specification" (E2M1 elements,
// E8M0 scale, blocks of 32) and "Conversion rules" (scale = 2^floor(log2 amax)
// / 4, round-to-nearest-even with saturation).  Random bits: Philox4x32-10 of
// Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/mxfp4.h"

namespace mxfp4 {

// ---------------------------------------------------------------------------
// Host/device layout helpers
// ---------------------------------------------------------------------------

// K-blocks of one MMA scale atom row group and the atom geometry: 128 rows x
// 4 K-blocks, 512 bytes, (row % 32) * 16 + ((row % 128) / 32) * 4 + kb % 4.
__host__ __device__ __forceinline__ int64_t mma_katoms(int64_t k) { return (k / 32 + 3) / 4; }

__host__ __device__ __forceinline__ int64_t mma_scale_off(int64_t row, int64_t kb, int64_t katoms) {
    return (((row >> 7) * katoms + (kb >> 2)) << 9) + ((row & 31) << 4) + (((row >> 5) & 3) << 2) + (kb & 3);
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (SC'11): 10 rounds of two 32x32->64 multiplies; the high
// halves are xored with the odd counter words and the key, the key advances
// by the Weyl constants after every round.
// ---------------------------------------------------------------------------
struct U4 { uint32_t x, y, z, w; };

__device__ __forceinline__ U4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                            uint32_t k0, uint32_t k1) {
    constexpr uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    constexpr uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint64_t p0 = (uint64_t)M0 * c0;   // one widening multiply each
        const uint64_t p1 = (uint64_t)M1 * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        c0 = n0; c1 = (uint32_t)p1; c2 = n2; c3 = (uint32_t)p0;
        k0 += W0; k1 += W1;
    }
    return U4{c0, c1, c2, c3};
}

// Sign mask of the RHT diagonal for a seed: word 0 of the block with counter
// (0, 0, 0, 0x52485400).  Computed on the host too (same function body).
__host__ __device__ inline uint32_t rht_sign_mask_hd(uint64_t seed) {
    uint32_t c0 = 0, c1 = 0, c2 = 0, c3 = 0x52485400u;
    uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
    for (int r = 0; r < 10; ++r) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        c1 = (uint32_t)p1; c3 = (uint32_t)p0; c0 = n0; c2 = n2;
        k0 += 0x9E3779B9u; k1 += 0xBB67AE85u;
    }
    return c0;
}

// ---------------------------------------------------------------------------
// bf16 <-> fp32
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two fp32 -> packed bf16x2 (round to nearest even), a in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
    return r;
}

// Eight bf16 values (a uint4, element 0 in the low half of .x) to fp32.
__device__ __forceinline__ void unpack_bf16x8(const uint4 &u, float *w) {
    w[0] = bf16lo(u.x); w[1] = bf16hi(u.x); w[2] = bf16lo(u.y); w[3] = bf16hi(u.y);
    w[4] = bf16lo(u.z); w[5] = bf16hi(u.z); w[6] = bf16lo(u.w); w[7] = bf16hi(u.w);
}

// max(|a|, |b|) of two bf16 pairs, NaN if either operand is NaN; the sign
// bits of the result are the operands' sign xor, not used here.
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// amax of 32 bf16 values packed in four uint4, as fp32 (exact: a maximum of
// bf16 magnitudes needs no rounding); NaN if any value is NaN.
__device__ __forceinline__ float amax_bf16x32(const uint4 *u) {
    const uint32_t a = bf16x2_absmax(bf16x2_absmax(u[0].x, u[0].y), bf16x2_absmax(u[0].z, u[0].w));
    const uint32_t b = bf16x2_absmax(bf16x2_absmax(u[1].x, u[1].y), bf16x2_absmax(u[1].z, u[1].w));
    const uint32_t c = bf16x2_absmax(bf16x2_absmax(u[2].x, u[2].y), bf16x2_absmax(u[2].z, u[2].w));
    const uint32_t d = bf16x2_absmax(bf16x2_absmax(u[3].x, u[3].y), bf16x2_absmax(u[3].z, u[3].w));
    const uint32_t m = bf16x2_absmax(bf16x2_absmax(a, b), bf16x2_absmax(c, d)) & 0x7FFF7FFFu;
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(bf16lo(m)), "f"(bf16hi(m)));
    return r;
}

// ---------------------------------------------------------------------------
// amax with NaN propagation (max.NaN returns NaN if either input is NaN)
// ---------------------------------------------------------------------------
__device__ __forceinline__ float amax_nan(float acc, float v) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(acc), "f"(fabsf(v)));
    return r;
}
// Two values at once: the three-input max of sm_100 (the same result as two
// nested max.NaN).
__device__ __forceinline__ float amax_nan2(float acc, float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(acc), "f"(fabsf(a)), "f"(fabsf(b)));
    return r;
}

// E8M0 scale code of a block from its amax (NaN or Inf -> 0xFF; 0 -> 0):
// clamp(floor(log2 amax) - 2 + 127, 0, 254).  For a normal amax the biased
// exponent field E gives floor(log2 amax) = E - 127, so the code is E - 2;
// a subnormal amax (E = 0) or E <= 2 clamps to 0.
__device__ __forceinline__ uint32_t scale_code_from_amax(float amax) {
    const uint32_t b = __float_as_uint(amax);
    if (b >= 0x7F800000u) return 0xFFu;
    const int e = (int)(b >> 23) - 2;
    return e > 0 ? (uint32_t)e : 0u;
}

// Scale code under the round-up rule: the smallest e with 6 * 2^e >= amax.
// With amax = 1.m * 2^(E - 127), amax / 2^(E - 129) = 4 * 1.m, which exceeds 6
// exactly when the mantissa field is above 0x400000 (1.m > 1.5).
__device__ __forceinline__ uint32_t scale_code_roundup(float amax) {
    const uint32_t b = __float_as_uint(amax);
    if (b >= 0x7F800000u) return 0xFFu;
    const int e = (int)(b >> 23) - 2 + ((b & 0x007FFFFFu) > 0x00400000u ? 1 : 0);
    return e > 0 ? (uint32_t)min(e, 254) : 0u;
}

// Scale code of a block under a scale rule (MXFP4_SCALE_* >> 4): 0 the
// reference floor rule, 1 round-up, 2 the 3/4 pre-scale (floor exponent).
__device__ __forceinline__ uint32_t scale_code_rule(float amax, int rule) {
    return rule == 1 ? scale_code_roundup(amax) : scale_code_from_amax(amax);
}

// Element scaling: y / X, or (3/4 y) / X under the pre-scale rule, each
// product rounded in fp32 (the division by the power of two X is exact
// unless the result is subnormal).  The rule is tested once per group.
__device__ __forceinline__ void scale8(float *w, float inv, int rule) {
    if (rule == 2) {
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = __fmul_rn(__fmul_rn(w[i], 0.75f), inv);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = __fmul_rn(w[i], inv);
    }
}
__device__ __forceinline__ void scale_block32(float *v, float inv, int rule) {
#pragma unroll
    for (int q = 0; q < 4; ++q) scale8(v + 8 * q, inv, rule);
}

// 2^-(code - 127) as fp32 for code in [0, 252]: biased exponent 254 - code.
__device__ __forceinline__ float inv_scale_from_code(uint32_t code) {
    return __uint_as_float((254u - code) << 23);
}

// 2^(code - 127) as fp32 for code in [0, 254] (code 0 is the subnormal 2^-127).
__device__ __forceinline__ float scale_from_code(uint32_t code) {
    return code ? __uint_as_float(code << 23) : __uint_as_float(0x00400000u);
}

// ---------------------------------------------------------------------------
// E2M1 encoders
// ---------------------------------------------------------------------------

// Eight scaled fp32 values -> 8 nibbles (round to nearest even, saturate to
// +-6), element 0 in bits 3:0.  cvt.rn.satfinite.e2m1x2.f32 d, a, b puts a in
// the high nibble and b in the low nibble of d.
__device__ __forceinline__ uint32_t e2m1x8_rn(const float *v) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// Right shift with the PTX rule for large amounts: a count of 32 or more (a
// negative int passed as unsigned included) gives 0.
__device__ __forceinline__ uint32_t shr_sat(uint32_t a, uint32_t n) {
    uint32_t d;
    asm("shr.u32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(n));
    return d;
}

// E2M1 code (bit 3 the sign) -> fp32, exact.  Bit pattern of an E2M1 magnitude code m (0..7): m >= 2 -> (252 + m) << 22
// (1.0 .. 6.0), m == 1 -> 0.5, m == 0 -> 0.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
    const uint32_t m = c & 7u;
    uint32_t b = m >= 2u ? (252u + m) << 22 : (m ? 0x3F000000u : 0u);
    b |= (c & 8u) << 28;
    return __uint_as_float(b);
}

// Sign bits of 8 values as the sign bits (bit 3) of 8 packed E2M1 nibbles:
// byte permutes with sign replication gather the even and the odd elements,
// a select interleaves them.
__device__ __forceinline__ uint32_t prmt_sign2(float a, float b) {
    uint32_t d;    // byte 0 = sign(a) replicated, byte 1 = sign(b) replicated
    asm("prmt.b32 %0, %1, %2, 0x00FB;" : "=r"(d) : "r"(__float_as_uint(a)), "r"(__float_as_uint(b)));
    return d;
}
__device__ __forceinline__ uint32_t prmt_lo2(uint32_t a, uint32_t b) {
    uint32_t d;    // bytes 0, 1 of a, then bytes 0, 1 of b
    asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t sign_nibbles8(const float *w) {
    const uint32_t ev = prmt_lo2(prmt_sign2(w[0], w[2]), prmt_sign2(w[4], w[6]));
    const uint32_t od = prmt_lo2(prmt_sign2(w[1], w[3]), prmt_sign2(w[5], w[7]));
    return ((ev & 0x0F0F0F0Fu) | (od & 0xF0F0F0F0u)) & 0x88888888u;
}

// Stochastic rounding of one clamped magnitude (bits ab, 0 <= |v| <= 6) as a
// fixed-point add.  With s = min(e - 117, 10) >= 0 (|v| >= 2^-10), the 64-bit
// number W * 2^s has the index of the grid point below |v| in its high word
// and f * 2^32 (f the position between the two neighbours, the SR threshold)
// in its low word; W is the 24-bit significand m below 1 and
// ab - (126 << 23) = ((e - 126) << 23) | mantissa from 1 up (grid steps 1 and
// 2 above 2 shift the index by 2 per binade), i.e. max(ab - 0x3F000000, m).
// Adding ~r carries into the high word exactly when r < f * 2^32, so the high
// word of W * 2^s + ~r is the rounded code.  Integer work: two add-min/max,
// one shift, one mask; the multiply-add runs on the FMA pipe.
__device__ __forceinline__ int32_t sr_shift(uint32_t ab) {
    return __viaddmin_s32((int32_t)(ab >> 23), -117, 10);
}
__device__ __forceinline__ uint32_t e2m1_sr_fixed(uint32_t ab, int32_t s, uint32_t nr) {
    const uint32_t m = (ab & 0x007FFFFFu) | 0x00800000u;
    const uint32_t w = (uint32_t)__viaddmax_s32((int32_t)ab, -0x3F000000, (int32_t)m);
    uint32_t p;    // 2^s; shl clamps a shift past 32 (s < 0 is never used)
    asm("shl.b32 %0, %1, %2;" : "=r"(p) : "r"(1u), "r"(s));
    return (uint32_t)(((uint64_t)w * p + nr) >> 32);
}

// Eight scaled values to eight packed E2M1 codes by stochastic rounding.  The
// random words are those of the Philox blocks b0 (elements 0-3) and b0 + 1
// (elements 4-7) under the key (k0, k1).  Magnitudes take the fixed-point add
// and are packed by a multiply-add chain (the nibbles do not overlap); signs
// go in at once.  A group holding a magnitude under 2^-10 (or a zero) adds
// the round-up bits of those magnitudes afterwards.
// Round-up bits of the magnitudes under 2^-10 in a group of eight.  The
// fixed-point add gives them code 0; the exact rule rounds such a value up to
// 0.5 when r < ceil(m * 2^(e - 117)) (m its 24-bit significand, e its biased
// exponent).  The random words are regenerated one Philox block at a time.
__device__ __forceinline__ uint32_t e2m1x8_sr_tiny(const float *w, uint64_t b0, uint32_t k0, uint32_t k1) {
    uint32_t up = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint64_t b = b0 + h;
        const U4 r = philox4x32_10((uint32_t)b, (uint32_t)(b >> 32), 0u, 0u, k0, k1);
        const uint32_t rr[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t ab = __float_as_uint(fminf(fabsf(w[4 * h + j]), 6.0f));
            const uint32_t e = ab >> 23;
            const uint32_t m = (ab & 0x007FFFFFu) | 0x00800000u;
            const uint32_t t = shr_sat(m - 1u, 117u - e) + 1u;
            if (ab - 1u < 0x3A7FFFFFu && rr[j] < t) up |= 1u << (4 * (4 * h + j));
        }
    }
    return up;
}

__device__ __forceinline__ uint32_t e2m1x8_sr(const float *w, uint64_t b0, uint32_t k0, uint32_t k1) {
    const uint64_t b1 = b0 + 1;
    const uint32_t sgn = sign_nibbles8(w);
    uint32_t mag = 0;
    int32_t any = 0;
    {
        const U4 r0 = philox4x32_10((uint32_t)b0, (uint32_t)(b0 >> 32), 0u, 0u, k0, k1);
        const U4 r1 = philox4x32_10((uint32_t)b1, (uint32_t)(b1 >> 32), 0u, 0u, k0, k1);
        const uint32_t rr[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
        for (int i = 7; i >= 0; --i) {
            const uint32_t ab = __float_as_uint(fminf(fabsf(w[i]), 6.0f));
            const int32_t sh = sr_shift(ab);
            any |= sh;
            mag = mag * 16u + e2m1_sr_fixed(ab, sh, ~rr[i]);
        }
    }
    if (__builtin_expect(any < 0, 0)) mag |= e2m1x8_sr_tiny(w, b0, k0, k1);
    return mag | sgn;
}

// ---------------------------------------------------------------------------
// In-register fast Walsh-Hadamard butterfly over D values, stages h = 1..D/2,
// (a, b) -> (a + b, a - b), each rounded in fp32.
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void fwht(float *v) {
#pragma unroll
    for (int h = 1; h < D; h <<= 1) {
#pragma unroll
        for (int i = 0; i < D; ++i) {
            if ((i & h) == 0) {
                const float a = v[i], b = v[i + h];
                v[i] = __fadd_rn(a, b);
                v[i + h] = __fsub_rn(a, b);
            }
        }
    }
}

template <int D>
__device__ __forceinline__ float rht_norm() {
    return D == 16 ? 0.25f : __uint_as_float(0x3E3504F3u);  // fp32(1/sqrt(32))
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  Every kernel of this library is launched
// with the programmatic-stream-serialization attribute, so its CTAs may start
// while the previous kernel on the stream is still draining.  Each kernel
// therefore executes pdl_wait() (griddepcontrol.wait: the previous grid has
// completed and its writes are visible) before its first global-memory read
// or write, and pdl_trigger() once its own CTAs are running, which lets the
// next kernel's launch and prologue overlap this one's tail.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace mxfp4

