/*
 * mxfp4_oracle.c -- plain, slow CPU oracle for the MXFP4 quantizer and the
 * MXFP4 block-scaled GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only tests/, the smoke check in __graft_entry__.py and the CPU
 * baseline leg of bench.py use it.  It shares no code, header, table or
 * constant generator with the CUDA library; the CUDA side never reads it.
 *
 * Sources (cited by page title and section):
 *  [MX-FMT]   "MXFP4" (aiwiki.ai), section "Format specification": E2M1
 *             element (1 sign, 2 exponent, 1 mantissa bit, bias 1, max 6,
 *             subnormal 0.5, no Inf/NaN), E8M0 scale (bias 127, exponents
 *             -127..127, 0xFF = NaN, no zero/Inf), block k = 32, 136 bits per
 *             block; the bit-pattern table of the eight E2M1 magnitudes; a NaN
 *             scale makes the whole block NaN.
 *  [MX-CONV]  same page, "Conversion rules": X = (largest power of two not
 *             above max|Vi|) / 4, each Vi/X quantized to FP4 with
 *             round-to-nearest-ties-to-even and saturation to +-6.  Dot
 *             product: C = X(A) X(B) sum_i Pi(A) Pi(B), blocks summed, FP32
 *             result, internal order left free.
 *  [MX-CLIP]  same page, "Clipping in the reference algorithm": shared
 *             exponent = floor(log2 amax) - 2; worked example amax 7.5 -> X = 1
 *             -> 7.5 stored as 6.
 *  [MX-TRAIN] same page, "Training with MXFP4" (table and the paragraph after
 *             it): stochastic rounding for unbiased gradients, random Hadamard
 *             transform against block outliers, Hadamard size 32 for MXFP4.
 *  [MX-GPTOSS] same page, "Use in models / gpt-oss": blocks along the last
 *             dimension, two FP4 values per uint8, scales stored apart.
 *  [ALTO]     "Training an MoE LLM in MXFP4: How We Closed the Gap to BF16"
 *             (thesingularityreport.com), abstract: hybrid 1D/2D block
 *             quantization, randomized Hadamard transforms and stochastic
 *             rounding on GPT-OSS-20B.
 *  [MX-NV]    same page, "Comparison with NVFP4": E2M1 elements in blocks of
 *             16, an FP8 E4M3 block scale (fractional, fitted to each block),
 *             a second-level FP32 scale per tensor, 4.5 bits per value.
 *  [PHILOX]   Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
 *             1, 2, 3", SC'11: the Philox4x32-10 counter-based generator.
 *
 * Readings where the pages are silent or ambiguous (each is restated where it
 * is used):
 *  R1  Inputs are bf16 bit patterns; bf16 -> fp32 is exact (16-bit shift).
 *  R2  RHT: y = c_d * H_d * diag(s) * x on each d-element segment (d = 16 or
 *      32) along the quantization axis (the last dimension for 1D-row and 2D
 *      blocks, dimension 0 for 1D-column blocks).  H_d is the Sylvester
 *      Hadamard matrix; it is applied as an in-place butterfly in fp32 with
 *      stages h = 1, 2, 4, ..., d/2, each pair (a, b) -> (a + b, a - b)
 *      rounded to nearest, then one fp32 multiply by c_16 = 0.25 or
 *      c_32 = fp32(1/sqrt(32)).  The sign s_j is -1 when bit j of the first
 *      Philox word for key = seed, counter = (0, 0, 0, 0x52485400) is set.
 *  R3  A block whose values contain a NaN, or whose amax is +Inf, gets scale
 *      code 0xFF and element codes 0.
 *  R4  amax == 0 gives scale code 0 and every element +-0.
 *  R5  The scale code is clamp(floor(log2 amax) - 2 + 127, 0, 254).
 *  R6  "Flush values below the smallest subnormal to zero" is read as the
 *      result of round-to-nearest-even on the full grid: |v| <= 0.25 gives 0,
 *      (0.25, 0.75) gives 0.5.
 *  R7  The sign bit of an element code is the sign of the scaled value, so a
 *      negative value that rounds to zero is stored as -0 (code 0x8).
 *  R8  Stochastic rounding: with lo <= |v| <= hi adjacent grid values and
 *      f = (|v| - lo) / (hi - lo), round up iff r < f * 2^32 where r is the
 *      32-bit Philox word for the element: word (g mod 4) of
 *      Philox4x32-10(key = seed, counter = (g/4 low, g/4 high, 0, 0)), g the
 *      linear index of the element in the quantized (output) view plus a
 *      caller-supplied offset.  |v| is clamped to 6 first.
 *  R9  Packing: byte j of a 32-element block holds element 2j in bits 3:0
 *      and element 2j+1 in bits 7:4.
 *  R10 2D blocks are 32x32 tiles of the [rows, cols] tensor; the optional
 *      transposed copy stores element (r, c) at row c, position r.
 *  R16 NVFP4 [MX-NV] (the page gives the format, not the scale rule): tensor
 *      scale S = fp32(amax_tensor / 2688), 2688 = 6 * 448 so the largest
 *      block scale is E4M3's maximum; block scale code = E4M3 nearest-even of
 *      fp32(amax_block / fp32(6 S)), saturating at 448; element divisor
 *      X = fp32(decode(code) * S); elements fp32(x / X) rounded to E2M1 (RNE
 *      or SR as R8).  A block whose scale rounds to 0 stores +-0; a tensor
 *      with amax 0 stores zeros; a NaN or Inf in the tensor makes every
 *      block scale NaN (0x7F) with codes 0.  E4M3 is the OCP FP8 format:
 *      bias 7, 3 mantissa bits, subnormals m * 2^-9, no Inf, 0x7F = NaN.
 *      Blocks run along the last dimension (1D row) or dimension 0 (1D
 *      column, transposed output), as for MXFP4; no RHT.
 *  R14 Scale rules besides R5 ([MX-CLIP] and the [MX-TRAIN] table):
 *      round-up: the decode scale amax / 6 rounded up to a power of two, that
 *        is the smallest e with 6 * 2^e >= amax, so no element saturates;
 *      3/4 pre-scale: the block exponent comes from the unscaled amax as in
 *        R5, and each element is multiplied by 3/4 in fp32 before the
 *        division by X, so no element reaches the clipping range.  The codes
 *        hold 3/4 of the values; the consumer undoes the factor.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fopenmp.  No FMA
 * contraction and no fast-math, so every float operation rounds as written.
 *
 * Mutation testing: building with -DORC_MUTANT=k (k >= 1) plants the k-th of
 * the numbered plausible mistakes marked MUT(k) below (a wrong tie rule, an
 * off-by-one exponent, swapped nibbles, ...).  tests/test_oracle_mutants.py
 * builds each one and checks that the pins fail on it.  Normal builds leave
 * ORC_MUTANT at 0, where every MUT(k) is the constant 0.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>

#ifndef ORC_MUTANT
#define ORC_MUTANT 0
#endif
#define MUT(k) (ORC_MUTANT == (k))

#define ORC_LAYOUT_1D_ROW 0
#define ORC_LAYOUT_1D_COL 1
#define ORC_LAYOUT_2D 2
#define ORC_ROUND_RNE 0
#define ORC_ROUND_SR 1
#define ORC_SCALE_FLOOR 0
#define ORC_SCALE_ROUNDUP 1
#define ORC_SCALE_PRESCALE_34 2

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 [PHILOX].  Round function: two 32x32->64 products of the    */
/* even counter words with the multipliers; the high halves are xored with   */
/* the odd counter words and the key; the key is bumped by the Weyl          */
/* constants between rounds.                                                 */
/* ------------------------------------------------------------------------ */
static const uint32_t PHILOX_M0 = 0xD2511F53u;
static const uint32_t PHILOX_M1 = 0xCD9E8D57u;
static const uint32_t PHILOX_W0 = 0x9E3779B9u;
static const uint32_t PHILOX_W1 = 0xBB67AE85u;

void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < (MUT(10) ? 9 : 10); ++round) {
        uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += PHILOX_W0;
        k1 += PHILOX_W1;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* R8: the random word for element index g. */
uint32_t orc_sr_word(uint64_t seed, uint64_t g)
{
    uint64_t blk = g >> 2;
    uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), 0u, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t w[4];
    orc_philox4x32_10(ctr, key, w);
    return w[g & 3];
}

/* R8: n consecutive stream words starting at index g0. */
void orc_sr_words(uint64_t seed, uint64_t g0, int64_t n, uint32_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_sr_word(seed, g0 + (uint64_t)i);
}

/* R2: the sign mask of the RHT diagonal. */
uint32_t orc_rht_sign_mask(uint64_t seed)
{
    uint32_t ctr[4] = {MUT(5) ? 0x52485400u : 0u, 0u, 0u, MUT(5) ? 0u : 0x52485400u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t w[4];
    orc_philox4x32_10(ctr, key, w);
    return w[0];
}

/* ------------------------------------------------------------------------ */
/* Number formats [MX-FMT].                                                  */
/* ------------------------------------------------------------------------ */

/* The eight non-negative E2M1 magnitudes, in code order 0b000..0b111, as in
 * the page's bit-pattern table (0 00 0 = 0, 0 00 1 = 0.5, ..., 0 11 1 = 6). */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Decode one 4-bit code: bit 3 is the sign. */
double orc_e2m1_decode(uint32_t code)
{
    double m = E2M1_MAG[code & 7u];
    return (code & 8u) ? -m : m;
}

/* Decode one E8M0 scale byte: 2^(code - 127); 0xFF is NaN. */
double orc_e8m0_decode(uint32_t code)
{
    if ((code & 0xFFu) == 0xFFu) return NAN;
    return ldexp(1.0, (int)(code & 0xFFu) - (MUT(15) ? 128 : 127));
}

/* R1: bf16 bit pattern -> fp32 (exact). */
float orc_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp32 -> bf16 with round-to-nearest-even (used only for bf16 outputs). */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    if (MUT(27)) u += 0x8000u;                 /* ties away from zero */
    else if (!MUT(28)) u += 0x7FFFu + lsb;     /* MUT(28): truncation */
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* Scale rule [MX-CONV], [MX-CLIP]; readings R3, R4, R5.                     */
/* Returns the E8M0 code for a block with the given amax (amax >= 0 or NaN). */
/* ------------------------------------------------------------------------ */
uint32_t orc_scale_code(float amax)
{
    if (isnan(amax) || isinf(amax)) return 0xFFu;   /* R3 */
    if (amax == 0.0f) return 0u;                    /* R4 */
    int ex;
    /* amax = m * 2^ex with m in [0.5, 1): floor(log2 amax) = ex - 1, exact
     * also for subnormal amax. */
    (void)frexpf(amax, &ex);
    int e = (ex - 1) - (MUT(2) ? 1 : 2);            /* [MX-CLIP] */
    int code = e + 127;
    if (code < 0) code = 0;                         /* R5 */
    if (code > 254) code = 254;
    return (uint32_t)code;
}

/* R14: the scale code under one of the three rules. */
uint32_t orc_scale_code_rule(float amax, int rule)
{
    if (rule != ORC_SCALE_ROUNDUP) return orc_scale_code(amax);
    if (isnan(amax) || isinf(amax)) return 0xFFu;
    if (amax == 0.0f) return 0u;
    int ex;
    (void)frexpf(amax, &ex);
    int e = (ex - 1) - 2;                           /* amax / 2^e in [4, 8) */
    /* the smallest e with 6 * 2^e >= amax: one more when amax / 2^e > 6 */
    if ((double)amax > (MUT(21) ? 5.0 : 6.0) * ldexp(1.0, e)) e += 1;
    int code = e + 127;
    if (code < 0) code = 0;
    if (code > 254) code = 254;
    return (uint32_t)code;
}

/* ------------------------------------------------------------------------ */
/* Element conversion [MX-CONV]; readings R6, R7, R8.                        */
/* ------------------------------------------------------------------------ */

/* Round-to-nearest-ties-to-even onto the E2M1 grid with saturation: the
 * nearest of the eight magnitudes; on an exact tie the even code wins. */
uint32_t orc_e2m1_rne(float v)
{
    uint32_t sign = (MUT(6) ? v < 0.0f : signbit(v)) ? 8u : 0u;   /* R7 */
    double a = fabs((double)v);
    if (a > 6.0) return sign | 7u;                  /* saturation */
    int best = 0;
    double best_d = fabs(a - E2M1_MAG[0]);
    for (int i = 1; i < 8; ++i) {
        double d = fabs(a - E2M1_MAG[i]);
        if (d < best_d || (d == best_d && (MUT(1) || ((i & 1) == 0 && (best & 1) == 1)))) {
            best = i;
            best_d = d;
        }
    }
    return sign | (uint32_t)best;
}

/* Stochastic rounding (R8): up with probability f, decided by r < f * 2^32. */
uint32_t orc_e2m1_sr(float v, uint32_t r)
{
    uint32_t sign = signbit(v) ? 8u : 0u;           /* R7 */
    double a = fabs((double)v);
    if (a > 6.0) a = 6.0;
    int lo = 0;
    for (int i = 0; i < 8; ++i)
        if (E2M1_MAG[i] <= a) lo = i;
    if (lo == 7 || E2M1_MAG[lo] == a) return sign | (uint32_t)lo;
    double f = (a - E2M1_MAG[lo]) / (E2M1_MAG[lo + 1] - E2M1_MAG[lo]);
    int up = (double)r < f * (MUT(3) ? 2147483648.0 : 4294967296.0);
    return sign | (uint32_t)(lo + up);
}

/* ------------------------------------------------------------------------ */
/* Randomized Hadamard transform [MX-TRAIN]; reading R2.                     */
/* ------------------------------------------------------------------------ */

static float rht_norm(int d)
{
    /* c_16 = 1/4 exactly; c_32 = 1/sqrt(32) rounded to fp32. */
    if (MUT(11)) return 1.0f;
    return d == 16 ? 0.25f : (float)(1.0 / sqrt(32.0));
}

/* Butterfly H_d in place, fixed stage order, fp32 rounding at every add. */
void orc_fwht_f32(float *v, int d)
{
    for (int h = 1; h < d; h <<= 1) {
        for (int i = 0; i < d; ++i) {
            if (i & h) continue;
            float a = v[i], b = v[i + h];
            v[i] = a + b;
            v[i + h] = MUT(16) ? b - a : a - b;
        }
    }
}

/* y = c_d * H_d * diag(s) * x. */
void orc_rht_forward(float *v, int d, uint32_t sign_mask)
{
    for (int j = 0; j < d; ++j)
        if ((sign_mask >> j) & 1u) v[j] = -v[j];
    orc_fwht_f32(v, d);
    float c = rht_norm(d);
    for (int j = 0; j < d; ++j) v[j] = v[j] * c;
}

/* x = diag(s) * H_d * (c_d * y): the inverse, since H_d H_d = d I and
 * c_d^2 d = 1 (up to the rounding of c_32). */
void orc_rht_inverse(float *v, int d, uint32_t sign_mask)
{
    orc_fwht_f32(v, d);
    float c = rht_norm(d);
    for (int j = 0; j < d; ++j) v[j] = v[j] * c;
    for (int j = 0; j < d; ++j)
        if ((sign_mask >> j) & 1u) v[j] = -v[j];
}

/* ------------------------------------------------------------------------ */
/* One MX block: scale and element codes from the (already transformed)      */
/* fp32 values.  n = 32 (1D) or 1024 (2D).  g[i] is the stream index of      */
/* element i (used by SR only).                                              */
/* ------------------------------------------------------------------------ */
static uint32_t quantize_block(const float *y, int n, int rnd, int rule, uint64_t seed,
                               const uint64_t *g, uint8_t *codes4)
{
    float amax = 0.0f;
    int has_nan = 0;
    for (int i = 0; i < n; ++i) {
        if (isnan(y[i])) has_nan = 1;
        float a = MUT(13) ? y[i] : fabsf(y[i]);
        if (MUT(22) && rule == ORC_SCALE_PRESCALE_34) a = 0.75f * a;
        if (a > amax) amax = a;
    }
    uint32_t sc = (has_nan && !MUT(9)) ? 0xFFu : orc_scale_code_rule(amax, rule);
    if (sc == 0xFFu) {                               /* R3 */
        for (int i = 0; i < n; ++i) codes4[i] = 0;
        return sc;
    }
    int e = (int)sc - 127;
    for (int i = 0; i < n; ++i) {
        /* R14: the 3/4 pre-scale is one fp32 multiply before the division by X */
        float vi = rule == ORC_SCALE_PRESCALE_34 ? 0.75f * y[i] : y[i];
        float v = ldexpf(vi, -e);                    /* Vi / X, exact or gradual underflow */
        codes4[i] = (uint8_t)(rnd == ORC_ROUND_SR ? orc_e2m1_sr(v, orc_sr_word(seed, g[i]))
                                                  : orc_e2m1_rne(v));
    }
    return sc;
}

static void put_nibble(uint8_t *row, int64_t pos, uint32_t code)
{
    uint8_t *b = row + (pos >> 1);
    if ((pos & 1) ^ MUT(4)) *b = (uint8_t)((*b & 0x0Fu) | (code << 4));   /* R9 */
    else *b = (uint8_t)((*b & 0xF0u) | (code & 0x0Fu));
}

uint32_t orc_get_nibble(const uint8_t *row, int64_t pos)
{
    uint8_t b = row[pos >> 1];
    return (pos & 1) ? (uint32_t)(b >> 4) : (uint32_t)(b & 0x0Fu);
}

/*
 * Quantize a bf16 tensor x[rows, cols] (row stride ld_x elements).
 *
 *  layout 1D_ROW: blocks of 32 along cols.  codes [rows, cols/2] (ld_codes
 *                 bytes), scales [rows, cols/32] (ld_scales bytes).
 *  layout 1D_COL: blocks of 32 along rows; the output is the transposed view:
 *                 codes [cols, rows/2], scales [cols, rows/32].
 *  layout 2D:     32x32 tiles.  codes [rows, cols/2], scales [rows/32,
 *                 cols/32]; if codes_t is given, also the transposed copy
 *                 codes_t [cols, rows/2] (ld_codes_t bytes).
 *
 * rht in {0, 16, 32}; rnd in {RNE, SR}; rule in {FLOOR, ROUNDUP,
 * PRESCALE_34} (R5, R14); the SR index of an element is its
 * linear index in the output view plus elem_offset.  Returns 0, or -1 on a
 * shape the format does not define.
 */
int orc_quantize_view(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld_x,
                      int layout, int rht, int rnd, int rule, uint64_t seed, uint64_t elem_offset,
                      int64_t sr_ld, uint8_t *codes, int64_t ld_codes, uint8_t *scales, int64_t ld_scales,
                      uint8_t *codes_t, int64_t ld_codes_t);

int orc_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld_x,
                 int layout, int rht, int rnd, int rule, uint64_t seed, uint64_t elem_offset,
                 uint8_t *codes, int64_t ld_codes, uint8_t *scales, int64_t ld_scales,
                 uint8_t *codes_t, int64_t ld_codes_t)
{
    return orc_quantize_view(x, rows, cols, ld_x, layout, rht, rnd, rule, seed, elem_offset, 0,
                             codes, ld_codes, scales, ld_scales, codes_t, ld_codes_t);
}

/*
 * As orc_quantize, for a tensor that is a slice of a larger one (R8: the SR
 * index is the element's position in the quantized output view of the WHOLE
 * tensor).  sr_ld is the row length of that whole output view (0: this
 * tensor's own, ocols); with elem_offset the index of the slice's first
 * element there, element (orow, ocol) of the slice draws index
 * orow * sr_ld + ocol + elem_offset.  A slice of tokens (rows of x) in the
 * 1D-column layout is a column range of the output view: sr_ld = the whole
 * tensor's rows, elem_offset = the slice's first row.
 */
int orc_quantize_view(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld_x,
                      int layout, int rht, int rnd, int rule, uint64_t seed, uint64_t elem_offset,
                      int64_t sr_ld, uint8_t *codes, int64_t ld_codes, uint8_t *scales, int64_t ld_scales,
                      uint8_t *codes_t, int64_t ld_codes_t)
{
    if (rht != 0 && rht != 16 && rht != 32) return -1;
    if (rule < ORC_SCALE_FLOOR || rule > ORC_SCALE_PRESCALE_34) return -1;
    uint32_t smask = rht ? orc_rht_sign_mask(seed) : 0u;

    if (layout == ORC_LAYOUT_1D_ROW || layout == ORC_LAYOUT_1D_COL) {
        /* Output view: orows x ocols, blocks along ocols. */
        int transposed = layout == ORC_LAYOUT_1D_COL;
        int64_t orows = transposed ? cols : rows;
        int64_t ocols = transposed ? rows : cols;
        int64_t gld = sr_ld ? sr_ld : ocols;            /* row length of the whole output view */
        if (ocols % 32) return -1;
        #pragma omp parallel for schedule(static)
        for (int64_t orow = 0; orow < orows; ++orow) {
            float y[32];
            uint64_t g[32];
            uint8_t c4[32];
            for (int64_t b = 0; b < ocols / 32; ++b) {
                for (int i = 0; i < 32; ++i) {
                    int64_t ocol = b * 32 + i;
                    int64_t r = transposed ? ocol : orow;
                    int64_t c = transposed ? orow : ocol;
                    y[i] = orc_bf16_to_f32(x[r * ld_x + c]);
                    g[i] = (uint64_t)(MUT(17) ? r * cols + c : orow * gld + ocol) + (MUT(12) ? 0 : elem_offset);
                }
                if (rht)
                    for (int s = 0; s < 32; s += rht) orc_rht_forward(y + s, rht, smask);
                uint32_t sc = quantize_block(y, 32, rnd, rule, seed, g, c4);
                scales[orow * ld_scales + b] = (uint8_t)sc;
                for (int i = 0; i < 32; ++i)
                    put_nibble(codes + orow * ld_codes, b * 32 + i, c4[i]);
            }
        }
        return 0;
    }
    if (layout == ORC_LAYOUT_2D) {
        if (rows % 32 || cols % 32) return -1;
        #pragma omp parallel for schedule(static)
        for (int64_t br = 0; br < rows / 32; ++br) {
            float y[1024];
            uint64_t g[1024];
            uint8_t c4[1024];
            for (int64_t bc = 0; bc < cols / 32; ++bc) {
                for (int i = 0; i < 32; ++i) {
                    int64_t r = br * 32 + i;
                    for (int j = 0; j < 32; ++j) {
                        int64_t c = bc * 32 + j;
                        y[i * 32 + j] = orc_bf16_to_f32(x[r * ld_x + c]);
                        g[i * 32 + j] = (uint64_t)(r * (sr_ld ? sr_ld : cols) + c) + elem_offset;
                    }
                    if (rht)
                        for (int s = 0; s < 32; s += rht) orc_rht_forward(y + i * 32 + s, rht, smask);
                }
                uint32_t sc = quantize_block(y, 1024, rnd, rule, seed, g, c4);
                scales[br * ld_scales + bc] = (uint8_t)sc;
                for (int i = 0; i < 32; ++i) {
                    int64_t r = br * 32 + i;
                    for (int j = 0; j < 32; ++j) {
                        int64_t c = bc * 32 + j;
                        put_nibble(codes + r * ld_codes, c, c4[i * 32 + j]);
                        if (codes_t) put_nibble(codes_t + c * ld_codes_t, MUT(8) ? r ^ 1 : r, c4[i * 32 + j]);
                    }
                }
            }
        }
        return 0;
    }
    return -1;
}

/*
 * Dequantize [MX-FMT]: value = decode(code) * 2^(scale - 127), NaN for a NaN
 * scale; then, if rht != 0, the inverse RHT on each segment along the block
 * axis.  Arguments mirror orc_quantize: for 1D_COL the codes/scales are the
 * transposed view and the output is written in the original [rows, cols]
 * orientation.  out_f32 (row stride ld_out) receives fp32 values; out_bf16
 * (same stride, may be NULL) receives them rounded to bf16.
 */
int orc_dequantize(const uint8_t *codes, int64_t ld_codes, const uint8_t *scales, int64_t ld_scales,
                   int64_t rows, int64_t cols, int layout, int rht, uint64_t seed,
                   float *out_f32, uint16_t *out_bf16, int64_t ld_out)
{
    if (rht != 0 && rht != 16 && rht != 32) return -1;
    uint32_t smask = rht ? orc_rht_sign_mask(seed) : 0u;
    int transposed = layout == ORC_LAYOUT_1D_COL;
    int64_t orows = transposed ? cols : rows;
    int64_t ocols = transposed ? rows : cols;
    if (ocols % 32) return -1;
    if (layout == ORC_LAYOUT_2D && (rows % 32)) return -1;
    #pragma omp parallel for schedule(static)
    for (int64_t orow = 0; orow < orows; ++orow) {
        float y[32];
        for (int64_t b = 0; b < ocols / 32; ++b) {
            /* MUT(29) reads a 2D tile's scale at the 1D row index (clamped to
             * the tile-row count, so the mistake stays inside the array). */
            int64_t srow = layout == ORC_LAYOUT_2D
                               ? (MUT(29) ? (orow < rows / 32 ? orow : rows / 32 - 1) : orow / 32)
                               : orow;
            uint8_t sc = scales[srow * ld_scales + b];
            double X = orc_e8m0_decode(sc);
            for (int i = 0; i < 32; ++i) {
                double v = orc_e2m1_decode(orc_get_nibble(codes + orow * ld_codes, b * 32 + i));
                y[i] = (float)(v * (MUT(14) ? 1.0 : X));   /* exact unless it overflows fp32 */
            }
            if (rht && !MUT(20))
                for (int s = 0; s < 32; s += rht) orc_rht_inverse(y + s, rht, smask);
            for (int i = 0; i < 32; ++i) {
                int64_t ocol = b * 32 + i;
                int64_t r = transposed ? (MUT(30) ? ocol ^ 1 : ocol) : orow;   /* MUT(30): nibble slip */
                int64_t c = transposed ? orow : ocol;
                out_f32[r * ld_out + c] = y[i];
                if (out_bf16) out_bf16[r * ld_out + c] = orc_f32_to_bf16(y[i]);
            }
        }
    }
    return 0;
}

/*
 * Block-scaled dot products [MX-CONV]: for C = A * B^T with both operands
 * stored K-major (row n of B holds the K values of output column n),
 *   C[m][n] = sum over K-blocks kb of 2^(ea + eb) * sum_{k in kb} a_k * b_k
 * in fp64, where a_k, b_k are E2M1 values and ea, eb the block exponents.
 * Each inner sum is a multiple of 1/4 no larger than 1152 in magnitude, so it
 * is exact; a NaN scale on either side makes the term (and C) NaN.
 * S[m][n] = sum_k |a_k 2^ea b_k 2^eb| (for the error bound), may be NULL.
 *
 * Scale addressing per operand (scale_mode): 0 = one scale per row and
 * K-block, [rows, K/32]; 1 = 2D tiles, [rows/32, K/32]; 2 = the 2D scales of
 * the transposed tensor, [K/32, rows/32].
 */
static double scale_at(const uint8_t *s, int64_t ld, int mode, int64_t row, int64_t kb)
{
    uint8_t code = mode == 0 ? s[row * ld + kb] : mode == 1 ? s[(row / 32) * ld + kb]
                                                            : s[kb * ld + row / 32];
    return orc_e8m0_decode(code);
}

void orc_gemm_entry(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, int64_t ld_as, int a_mode,
                    const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales, int64_t ld_bs, int b_mode,
                    int64_t K, int64_t m, int64_t n, double *c_out, double *s_out)
{
    double acc = 0.0, sabs = 0.0;
    for (int64_t kb = 0; kb < K / 32; ++kb) {
        double xa = scale_at(a_scales, ld_as, a_mode, m, kb);
        double xb = scale_at(b_scales, ld_bs, b_mode, n, kb);
        double dot = 0.0, dabs = 0.0;
        for (int i = 0; i < 32; ++i) {
            int64_t k = kb * 32 + i;
            double a = orc_e2m1_decode(orc_get_nibble(a_codes + m * lda, k));
            double b = orc_e2m1_decode(orc_get_nibble(b_codes + n * ldb, MUT(19) ? k ^ 1 : k));
            dot += a * b;
            dabs += fabs(a * b);
        }
        acc += (MUT(7) ? xa / xb : xa * xb) * dot;
        sabs += xa * xb * dabs;
    }
    *c_out = acc;
    if (s_out) *s_out = sabs;
}

void orc_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, int64_t ld_as, int a_mode,
              const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales, int64_t ld_bs, int b_mode,
              int64_t M, int64_t N, int64_t K, double *c, int64_t ldc, double *s, int64_t lds)
{
    #pragma omp parallel for schedule(dynamic, 4)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            orc_gemm_entry(a_codes, lda, a_scales, ld_as, a_mode, b_codes, ldb, b_scales, ld_bs, b_mode,
                           K, m, n, &c[m * ldc + n], s ? &s[m * lds + n] : NULL);
}

/* ======================================================================== */
/* NVFP4 [MX-NV], reading R16.                                                */
/* ======================================================================== */

/* E4M3 decode: (-1)^s (1 + m/8) 2^(e-7), subnormal m 2^-9, 0x7F/0xFF NaN. */
double orc_e4m3_decode(uint32_t code)
{
    code &= 0xFFu;
    int sgn = (int)(code >> 7), e = (int)((code >> 3) & 15u), m = (int)(code & 7u);
    if (e == 15 && m == 7) return NAN;
    double v = e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return sgn ? -v : v;
}

/* Nearest non-negative E4M3 code to a >= 0 (ties to the even code), by search
 * over the 127 non-negative finite values; saturates at 448 (code 0x7E). */
uint32_t orc_e4m3_rne(double a)
{
    if (a >= 448.0) return 0x7Eu;
    int best = 0;
    double bd = fabs(a);
    for (int c = 1; c < 0x7F; ++c) {
        double d = fabs(a - orc_e4m3_decode((uint32_t)c));
        if (d < bd || (d == bd && (MUT(24) ? (c & 1) == 1 : ((c & 1) == 0 && (best & 1) == 1)))) {
            best = c;
            bd = d;
        }
    }
    return (uint32_t)best;
}

/* Tensor scale S = amax / (6 * 448) in fp32. */
float orc_nvfp4_tensor_scale(float amax)
{
    return amax / (MUT(23) ? 1536.0f : 2688.0f);
}

/* One NVFP4 block of 16 values with tensor scale S: the scale code and the
 * element codes (g[i]: SR stream index of element i). */
static uint32_t nv_block(const float *y, float S, int rnd, uint64_t seed, const uint64_t *g, uint8_t *c4)
{
    if (!isfinite(S)) {                                   /* NaN or Inf in the tensor */
        for (int i = 0; i < 16; ++i) c4[i] = 0;
        return 0x7Fu;
    }
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(y[i]);
        if (a > amax) amax = a;
    }
    uint32_t code = 0;
    if (S > 0.0f) {
        float six_s = 6.0f * S;
        float q = amax / six_s;
        code = orc_e4m3_rne((double)q);
    }
    float X = MUT(26) ? (float)orc_e4m3_decode(code) : (float)orc_e4m3_decode(code) * S;
    for (int i = 0; i < 16; ++i) {
        if (X == 0.0f) {                                  /* scale rounded to 0: +-0 */
            c4[i] = (uint8_t)orc_e2m1_rne(copysignf(0.0f, y[i]));
            continue;
        }
        float v = y[i] / X;
        c4[i] = (uint8_t)(rnd == ORC_ROUND_SR ? orc_e2m1_sr(v, orc_sr_word(seed, g[i])) : orc_e2m1_rne(v));
    }
    return code;
}

/* amax over a bf16 tensor, NaN if any element is NaN. */
static float nv_tensor_amax(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld_x)
{
    float amax = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            float v = orc_bf16_to_f32(x[r * ld_x + c]);
            if (isnan(v)) return NAN;
            if (fabsf(v) > amax) amax = fabsf(v);
        }
    return amax;
}

/*
 * NVFP4 quantize of x[rows, cols]: layout 1D_ROW (blocks of 16 along cols;
 * codes [rows, cols/2], scales [rows, cols/16]) or 1D_COL (blocks along rows,
 * transposed view: codes [cols, rows/2], scales [cols, rows/16]).  Writes the
 * tensor amax (the second-level scale is amax / 2688) to *tensor_amax.
 */
int orc_nvfp4_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld_x, int layout, int rnd,
                       uint64_t seed, uint64_t elem_offset, uint8_t *codes, int64_t ld_codes, uint8_t *scales,
                       int64_t ld_scales, float *tensor_amax)
{
    if (layout != ORC_LAYOUT_1D_ROW && layout != ORC_LAYOUT_1D_COL) return -1;
    int transposed = layout == ORC_LAYOUT_1D_COL;
    int64_t orows = transposed ? cols : rows;
    int64_t ocols = transposed ? rows : cols;
    if (ocols % 16) return -1;
    float amax_t = nv_tensor_amax(x, rows, cols, ld_x);
    *tensor_amax = amax_t;
    float S = isnan(amax_t) ? NAN : orc_nvfp4_tensor_scale(amax_t);
    #pragma omp parallel for schedule(static)
    for (int64_t orow = 0; orow < orows; ++orow) {
        float y[16];
        uint64_t g[16];
        uint8_t c4[16];
        for (int64_t b = 0; b < ocols / 16; ++b) {
            for (int i = 0; i < 16; ++i) {
                int64_t ocol = b * 16 + i;
                int64_t r = transposed ? ocol : orow;
                int64_t c = transposed ? orow : ocol;
                y[i] = orc_bf16_to_f32(x[r * ld_x + c]);
                g[i] = (uint64_t)(orow * ocols + ocol) + elem_offset;
            }
            scales[orow * ld_scales + b] = (uint8_t)nv_block(y, S, rnd, seed, g, c4);
            for (int i = 0; i < 16; ++i) put_nibble(codes + orow * ld_codes, b * 16 + i, c4[i]);
        }
    }
    return 0;
}

/* NVFP4 dequantize: value = fp32(fp32(decode(code) * decode(scale)) * S). */
int orc_nvfp4_dequantize(const uint8_t *codes, int64_t ld_codes, const uint8_t *scales, int64_t ld_scales,
                         int64_t rows, int64_t cols, int layout, float tensor_amax, float *out, int64_t ld_out)
{
    int transposed = layout == ORC_LAYOUT_1D_COL;
    int64_t orows = transposed ? cols : rows;
    int64_t ocols = transposed ? rows : cols;
    if (ocols % 16) return -1;
    float S = orc_nvfp4_tensor_scale(tensor_amax);
    for (int64_t orow = 0; orow < orows; ++orow)
        for (int64_t ocol = 0; ocol < ocols; ++ocol) {
            float sv = (float)orc_e4m3_decode(scales[orow * ld_scales + ocol / 16]);
            float e = (float)orc_e2m1_decode(orc_get_nibble(codes + orow * ld_codes, ocol));
            float v = (e * sv) * S;
            int64_t r = transposed ? ocol : orow, c = transposed ? orow : ocol;
            out[r * ld_out + c] = v;
        }
    return 0;
}

/* NVFP4 block dot products: C[m][n] = S_a S_b sum over 16-blocks of
 * s_a s_b sum a_k b_k in fp64; S[m][n] the matching sum of |terms|. */
void orc_nvfp4_gemm_entry(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, int64_t ld_as,
                          float a_amax, const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales,
                          int64_t ld_bs, float b_amax, int64_t K, int64_t m, int64_t n, double *c_out,
                          double *s_out)
{
    double acc = 0.0, sabs = 0.0;
    double ts = (double)orc_nvfp4_tensor_scale(a_amax) * (double)orc_nvfp4_tensor_scale(b_amax);
    for (int64_t kb = 0; kb < K / 16; ++kb) {
        double xa = orc_e4m3_decode(a_scales[m * ld_as + kb]);
        double xb = orc_e4m3_decode(b_scales[n * ld_bs + kb]);
        double dot = 0.0, dabs = 0.0;
        for (int i = 0; i < 16; ++i) {
            int64_t k = kb * 16 + i;
            double a = orc_e2m1_decode(orc_get_nibble(a_codes + m * lda, k));
            double b = orc_e2m1_decode(orc_get_nibble(b_codes + n * ldb, k));
            dot += a * b;
            dabs += fabs(a * b);
        }
        acc += xa * xb * dot;
        sabs += fabs(xa * xb) * dabs;
    }
    *c_out = MUT(25) ? acc : acc * ts;
    if (s_out) *s_out = sabs * fabs(ts);
}

/* Number of OpenMP threads the oracle runs with (1 without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
int orc_num_threads(void) { return omp_get_max_threads(); }
void orc_set_num_threads(int n) { omp_set_num_threads(n); }
#else
int orc_num_threads(void) { return 1; }
void orc_set_num_threads(int n) { (void)n; }
#endif
