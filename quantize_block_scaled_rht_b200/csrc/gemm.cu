// gemm.cu -- MXFP4 block-scaled GEMM (dense and grouped) for sm_100a.
//
// "MXFP4" (aiwiki.ai), "Conversion rules": the block dot product
// C = X(A) X(B) sum_i Pi(A) Pi(B), block products summed, FP32 result; the
// order of operations is the implementation's.  "Hardware support": Blackwell
// tensor cores apply MXFP4 block scales in hardware.  Here that is
// tcgen05.mma kind::mxf4.block_scale: E2M1 operands from shared memory, one
// UE8M0 scale per 32 K-elements from tensor memory, FP32 accumulators in
// tensor memory (TMEM), 64 K-elements per instruction.
//
// Kernel structure: persistent, clusters of two CTAs (one per SM) that share
// one 256 x BN output tile with the pair MMA (cta_group::2): each CTA holds 128
// rows of A and BN/2 rows of B, so every SM streams 128 + BN/2 operand rows per
// K step instead of 128 + BN.  Per CTA, 6 warps:
//   warp 0      TMA producer: its A rows, its half of B and the scale atoms
//               (A: its own 128 rows; B: all BN rows) into a STAGES-deep ring
//               (MXFP4: 3 stages of 512 K-elements); every load completes on
//               the even CTA's stage barrier;
//   warp 1      TMEM owner; in the even CTA also the MMA issuer: scale atoms
//               to TMEM (tcgen05.cp, both CTAs), 4 * KCH pair MMAs of K = 64
//               per stage into one of two accumulators, stage release by a
//               commit to both CTAs;
//   warps 2..5  epilogue: TMEM -> registers -> swizzled smem -> TMA store of
//               this CTA's 128 rows (FP32, or bf16 rounded to nearest even),
//               overlapping the next tile's MMAs, then an arrive on the even
//               CTA's accumulator-empty barrier.
// Every barrier wait is bounded by the GPU global timer; a wait that runs out
// records MXFP4_ERR_TIMEOUT, raises the CTA's abort flag, and each role drains
// what it has in flight before both CTAs meet at the final cluster barrier.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mxfp4 {

constexpr int BM = 128;                               // rows per CTA
constexpr int CHUNK = 128;                            // K bytes per swizzled chunk (256 E2M1 = 8 scale blocks)
constexpr int EPI_WARPS = 4;
constexpr int EPI_BUF = 32 * 32 * 4;                  // 32 rows x 32 FP32
constexpr int EPI_BYTES = EPI_WARPS * 2 * EPI_BUF;
constexpr int BAR_BYTES = 256;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_GROUPS = 1024;
constexpr int MAX_STAGES = 8;

// Tile configuration: a pair tile is 256 x BN; each stage of the STAGES-deep
// smem ring holds KCH chunks of K (KCH * 256 E2M1 elements, 4 * KCH MMAs).
// NV: NVFP4 operands (UE4M3 scales per 16 elements, kind::mxf4nvf4) instead of
// MXFP4 (UE8M0 per 32, kind::mxf4).  A scale atom holds 4 blocks of every row
// of a 128-row tile: 128 K-elements for MXFP4, 64 for NVFP4.
template <int BN_, int STAGES_, int KCH_, bool NV_ = false>
struct TileCfg {
    static constexpr int BN = BN_;
    static constexpr int STAGES = STAGES_;
    static constexpr int KCH = KCH_;
    static constexpr bool NV = NV_;
    static constexpr int KSTEP = 256 * KCH;           // E2M1 elements of K per stage
    static constexpr int KATOM = NV ? 64 : 128;       // K-elements per scale atom
    static constexpr int NATOM = KSTEP / KATOM;       // scale atoms per row tile per stage
    // B scale atoms span one 128-row tile when BN = 128, two when BN = 192
    // (a 192-column tile starts at 0 or 64 within a 128-row scale tile).
    static constexpr int NRT = BN == 128 ? 1 : 2;
    static constexpr int A_CHUNK = BM * CHUNK;               // 16 KB per chunk
    static constexpr int B_CHUNK = (BN / 2) * CHUNK;         // this CTA's half of the B tile
    static constexpr int A_BYTES = KCH * A_CHUNK;
    static constexpr int B_BYTES = KCH * B_CHUNK;
    static constexpr int SFA_BYTES = NATOM * 512;
    static constexpr int SFB_BYTES = NRT * NATOM * 512;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr uint32_t STAGE_TX = 2u * STAGE_BYTES;   // both CTAs complete on the even CTA's barrier
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;
    // TMEM columns (per CTA): accumulator 0 at [0, BN), the scale factors of
    // two consecutive stages after it, accumulator 1 at the top.
    static constexpr uint32_t SF_COL = BN;
    static constexpr uint32_t SF_STAGE_COLS = 4 * NATOM * (1 + NRT);
    static constexpr uint32_t ACC1_COL = TMEM_COLS - BN;
    // Instruction descriptor, kind::mxf4 block-scaled: A/B E2M1 (1), K-major,
    // N >> 3 at bit 17, UE8M0 scales (bit 23), M >> 4 at bit 24 (M = 256 for
    // the pair), scale-factor byte selectors at bits 4 (B) and 29 (A).
    static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                      ((NV ? 0u : 1u) << 23) | ((uint32_t)(256 >> 4) << 24);
    static_assert(BN == 128 || BN == 192, "tile width");
    static_assert(KCH == 1 || KCH == 2, "chunks per stage");
    static_assert(STAGES <= MAX_STAGES, "stages");
    static_assert(SF_COL + 2 * SF_STAGE_COLS <= ACC1_COL, "TMEM layout");
    static_assert(A_CHUNK % 1024 == 0 && B_CHUNK % 1024 == 0 && STAGE_BYTES % 1024 == 0, "swizzle alignment");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// Output of the epilogue: FP32, bf16 (nearest even), or MXFP4 (each 1D row
// block of 32 FP32 results requantized: amax, E8M0 scale, E2M1 RNE codes).
constexpr int OUT_F32 = 0, OUT_BF16 = 1, OUT_MX = 2;

using DefaultCfg = TileCfg<192, 3, 2>;
using NvCfg = TileCfg<192, 5, 1, true>;

__device__ unsigned int g_error_code;

__device__ __forceinline__ void record_error(unsigned int code) { atomicCAS(&g_error_code, 0u, code); }

struct GemmParams {
    int64_t M, N, K;
    int64_t katoms;            // ceil(K / 128): scale atoms per 128-row tile
    int64_t b_rowtiles;        // ceil(N / 128): 128-row scale tiles of one B operand
    void *c;                   // FP32, bf16 [.., ldc elements] or MXFP4 codes [.., ldc bytes]
    int64_t ldc;
    uint8_t *c_scales;         // MXFP4 output: scales, row-major [.., ld_c_scales] or GEMM-ready
    int64_t ld_c_scales, c_katoms;
    int c_scale_mma;
    const int32_t *group_offsets;
    const int32_t *group_sizes;
    const float *a_amax, *b_amax;   // NVFP4 tensor amaxes (second-level scales amax / 2688)
    int num_groups;
    uint64_t wait_limit_ns;
};

struct Shared {
    uint64_t full[MAX_STAGES], empty[MAX_STAGES];
    uint64_t tmem_full[2], tmem_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    volatile int abort;
    int drain_failed;    // set in both CTAs by the leader when a bounded drain wait ran out
    int ntiles;
};

// Mark the pair's drain as failed, in this CTA and in its peer (rank ^ 1).
__device__ __forceinline__ void mark_drain_failed(Shared *sh, uint32_t rank) {
    sh->drain_failed = 1;
    const uint32_t peer = mapa_shared(smem_u32(&sh->drain_failed), rank ^ 1u);
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer), "r"(1u) : "memory");
}

// Bounded wait: true once the phase of `parity` has completed; false if the
// CTA aborted or the wait ran past the limit (which records the timeout and
// aborts the CTA).  `hard` waits ignore the abort flag (used while draining).
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, Shared *sh, uint64_t limit,
                                           bool hard = false) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31u) == 0u) {
            if (!hard && sh->abort) return false;
            if (globaltimer_ns() - t0 > limit) {
                if (!hard) {
                    record_error(MXFP4_ERR_TIMEOUT);
                    sh->abort = 1;
                }
                return false;
            }
        }
    }
}

__device__ __forceinline__ void spin_ns(uint64_t ns) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < ns) {
    }
}

struct TileInfo {
    int64_t row0;       // first A row of this CTA's half
    int64_t c_row0;     // first C row of this CTA's half
    int rows_valid;     // rows of this CTA's half that belong to the problem (grouped: to the group)
    int64_t n0;         // first C column
    int64_t b_row;      // TMA row coordinate of the first B row of the pair tile
    int64_t sfb_rt_base;  // first 128-row scale tile of this B operand (expert)
    int64_t k0;         // first K element of the tile's reduction (grouped K: the group's offset)
    int64_t kg;         // K elements of the reduction
};

// Kernel modes: dense; grouped rows (per-expert row ranges of A, one B per
// expert); grouped K (per-expert K ranges of both operands, one C per expert).
constexpr int MODE_DENSE = 0, MODE_GROUPED_M = 1, MODE_GROUPED_K = 2;

// Pair tile t -> coordinates.  Dense: M in steps of 256 (fastest), then N.
// Grouped rows: group g owns cum[g+1] - cum[g] pair tiles.  Grouped K: group
// g owns tiles_m x tiles_n tiles of its [M, N] output over K range
// [cum[g], cum[g+1]) (cum holds the validated K offsets).
template <int BN, int MODE>
__device__ __forceinline__ TileInfo get_tile(int t, uint32_t rank, const GemmParams &p, const int *cum,
                                             int tiles_n) {
    TileInfo ti;
    ti.k0 = 0;
    ti.kg = p.K;
    if constexpr (MODE == MODE_GROUPED_K) {
        const int tiles_m = (int)((p.M + 255) / 256);
        const int g = t / (tiles_m * tiles_n), local = t - g * (tiles_m * tiles_n);
        const int tm = local % tiles_m, tn = local / tiles_m;
        ti.row0 = (int64_t)tm * 256 + 128 * rank;
        ti.c_row0 = (int64_t)g * p.M + ti.row0;
        const int64_t left = p.M - ti.row0;
        ti.rows_valid = left <= 0 ? 0 : (left < BM ? (int)left : BM);
        ti.n0 = (int64_t)tn * BN;
        ti.b_row = ti.n0;
        ti.sfb_rt_base = 0;
        ti.k0 = cum[g];
        ti.kg = (int64_t)cum[g + 1] - cum[g];
    } else if constexpr (MODE == MODE_DENSE) {
        const int tiles_m = (int)((p.M + 255) / 256);
        const int tm = t % tiles_m, tn = t / tiles_m;
        ti.row0 = (int64_t)tm * 256 + 128 * rank;
        const int64_t left = p.M - ti.row0;
        ti.rows_valid = left <= 0 ? 0 : (left < BM ? (int)left : BM);
        ti.n0 = (int64_t)tn * BN;
        ti.b_row = ti.n0;
        ti.sfb_rt_base = 0;
        ti.c_row0 = ti.row0;
    } else {
        int g = 0;
        while (g + 1 < p.num_groups && cum[g + 1] <= t) ++g;
        const int local = t - cum[g];
        const int tiles_g = (cum[g + 1] - cum[g]) / tiles_n;
        const int tm = local % tiles_g, tn = local / tiles_g;
        const int64_t size = p.group_sizes[g];
        const int64_t r_in = (int64_t)tm * 256 + 128 * rank;
        ti.row0 = (int64_t)p.group_offsets[g] + r_in;
        const int64_t left = size - r_in;
        ti.rows_valid = left <= 0 ? 0 : (left < BM ? (int)left : BM);
        ti.n0 = (int64_t)tn * BN;
        ti.b_row = (int64_t)g * p.N + ti.n0;
        ti.sfb_rt_base = (int64_t)g * p.b_rowtiles;
        ti.c_row0 = ti.row0;
    }
    return ti;
}

// One K stage of the pair tile, issued by the converged MMA warp: the stage's
// scale atoms go to tensor memory (A: NATOMS atoms of this pair's rows; B: NRT
// 128-row tiles x NATOMS atoms), then NK MMAs of K = 64 walk the 128-byte
// swizzled chunk rows 32 bytes at a time (4 MMAs per chunk).  The scale
// selector k & 1 picks bytes 0-1 or 2-3 of each 32-bit scale word (two
// 32-element blocks per MMA); k >> 1 steps to the next 4-block atom.
template <class Cfg, int NATOMS, int NK>
__device__ __forceinline__ void issue_stage(uint32_t d_tmem, uint32_t st, uint32_t sfa_col, uint32_t b_shift,
                                            bool first) {
    constexpr int NRT = Cfg::NRT, NATOM = Cfg::NATOM;
    const uint32_t sfb_col = sfa_col + 4u * NATOM;
    const uint64_t sf_desc = smem_desc(st + Cfg::A_BYTES + Cfg::B_BYTES, 0, 128, 0);
#pragma unroll
    for (int a = 0; a < NATOMS; ++a) {
        tc_cp_32x128_warpx4_pair_elect(sfa_col + 4u * a, sf_desc + (uint64_t)((512 * a) >> 4));
#pragma unroll
        for (int rt = 0; rt < NRT; ++rt)
            tc_cp_32x128_warpx4_pair_elect(sfb_col + 4u * NRT * a + 4u * rt,
                                           sf_desc + (uint64_t)((Cfg::SFA_BYTES + NATOM * 512 * rt + 512 * a) >> 4));
    }
    const uint64_t adesc = smem_desc(st, 16, 1024, 2);
    const uint64_t bdesc = smem_desc(st + Cfg::A_BYTES, 16, 1024, 2);
#pragma unroll
    for (int k = 0; k < NK; ++k) {
        const uint64_t a_off = (uint64_t)(((k >> 2) * Cfg::A_CHUNK + (k & 3) * 32) >> 4);
        const uint64_t b_off = (uint64_t)(((k >> 2) * Cfg::B_CHUNK + (k & 3) * 32) >> 4);
        if constexpr (Cfg::NV) {
            // one atom (4 scales of 16) per K = 64 instruction
            mma_nvf4_pair_elect(d_tmem, adesc + a_off, bdesc + b_off, Cfg::IDESC, sfa_col + 4u * (uint32_t)k,
                                sfb_col + 4u * NRT * (uint32_t)k + b_shift, (k == 0 && first) ? 0u : 1u);
        } else {
            const uint32_t idesc = (k & 1) ? (Cfg::IDESC | (2u << 29) | (2u << 4)) : Cfg::IDESC;
            mma_mxf4_pair_elect(d_tmem, adesc + a_off, bdesc + b_off, idesc, sfa_col + 4u * (uint32_t)(k >> 1),
                                sfb_col + 4u * NRT * (uint32_t)(k >> 1) + b_shift, (k == 0 && first) ? 0u : 1u);
        }
    }
}

// Partial last K stage (K not a multiple of the stage depth): NK = kleft / 64
// MMAs and ceil(NK / 2) scale atoms.
template <class Cfg>
__device__ __noinline__ void issue_stage_tail(uint32_t d_tmem, uint32_t st, uint32_t sfa_col, uint32_t b_shift,
                                              bool first, int nk) {
    if constexpr (Cfg::NV) {                  // one atom per MMA; a stage holds 4 * KCH MMAs
        switch (nk) {
            case 1: issue_stage<Cfg, 1, 1>(d_tmem, st, sfa_col, b_shift, first); break;
            case 2: issue_stage<Cfg, 2, 2>(d_tmem, st, sfa_col, b_shift, first); break;
            case 3: issue_stage<Cfg, 3, 3>(d_tmem, st, sfa_col, b_shift, first); break;
            default: break;
        }
        return;
    }
    switch (nk) {
        case 1: issue_stage<Cfg, 1, 1>(d_tmem, st, sfa_col, b_shift, first); break;
        case 2: issue_stage<Cfg, 1, 2>(d_tmem, st, sfa_col, b_shift, first); break;
        case 3: issue_stage<Cfg, 2, 3>(d_tmem, st, sfa_col, b_shift, first); break;
        case 4: issue_stage<Cfg, 2, 4>(d_tmem, st, sfa_col, b_shift, first); break;
        case 5: issue_stage<Cfg, 3, 5>(d_tmem, st, sfa_col, b_shift, first); break;
        case 6: issue_stage<Cfg, 3, 6>(d_tmem, st, sfa_col, b_shift, first); break;
        case 7: issue_stage<Cfg, 4, 7>(d_tmem, st, sfa_col, b_shift, first); break;
        default: break;   // a full stage never takes this path
    }
}

template <class Cfg, int MODE, int OUT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    mxfp4_gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                      const __grid_constant__ CUtensorMap tma_c, const __grid_constant__ CUtensorMap tma_sfa,
                      const __grid_constant__ CUtensorMap tma_sfb, const GemmParams p) {
    constexpr int BN = Cfg::BN, STAGES = Cfg::STAGES;
    constexpr int A_BYTES = Cfg::A_BYTES, B_BYTES = Cfg::B_BYTES, SFA_BYTES = Cfg::SFA_BYTES;
    constexpr int STAGE_BYTES = Cfg::STAGE_BYTES, KCH = Cfg::KCH, NATOM = Cfg::NATOM;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *stage_base = smem;
    uint8_t *epi_base = smem + STAGES * STAGE_BYTES;
    Shared *sh = reinterpret_cast<Shared *>(epi_base + EPI_BYTES);
    constexpr bool GROUPED = MODE == MODE_GROUPED_M;
    __shared__ int cum[MODE != MODE_DENSE ? MAX_GROUPS + 1 : 1];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();               // 0 = MMA issuer of the pair
    const int pair = (int)cluster_id_x(), npairs = (int)nclusters_x();
    const int tiles_n = (int)((p.N + BN - 1) / BN);
    auto ktiles_of = [](const TileInfo &ti) { return (int)((ti.kg + Cfg::KSTEP - 1) / Cfg::KSTEP); };
    const uint64_t limit = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(&sh->full[s], 1); mbar_init(&sh->empty[s], 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(&sh->tmem_full[b], 1); mbar_init(&sh->tmem_empty[b], 2 * EPI_WARPS); }
        mbar_init(&sh->drain, 1);
        sh->abort = 0;
        sh->drain_failed = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
        prefetch_tmap(&tma_a);
        prefetch_tmap(&tma_b);
        prefetch_tmap(&tma_c);
        prefetch_tmap(&tma_sfa);
        prefetch_tmap(&tma_sfb);
    }
    if (warp == 1) {
        tmem_alloc_pair(&sh->tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    // the prologue above touches no global memory; from here on the previous
    // kernel's outputs are read (operands, group offsets) and C is written
    pdl_wait();
    pdl_trigger();
    if constexpr (GROUPED) {
        if (threadIdx.x == 32 * 2) {
            int acc = 0;
            for (int g = 0; g < p.num_groups; ++g) {
                cum[g] = acc;
                const int64_t off = p.group_offsets[g], nxt = p.group_offsets[g + 1];
                const int64_t size = p.group_sizes[g];
                int tm = 0;
                if ((off % BM) != 0 || size < 0 || off + size > nxt || nxt > p.M) {
                    if (rank == 0) record_error(MXFP4_ERR_INVALID_ARG);
                } else {
                    tm = (int)((size + 255) / 256);
                }
                acc += tm * tiles_n;
            }
            cum[p.num_groups] = acc;
            sh->ntiles = acc;
        }
    } else if constexpr (MODE == MODE_GROUPED_K) {
        if (threadIdx.x == 32 * 2) {
            // K offsets: multiples of 128, non-decreasing, within K; a bad
            // entry records INVALID_ARG and empties the group
            int prev = 0;
            bool bad = false;
            for (int g = 0; g <= p.num_groups; ++g) {
                int o = p.group_offsets[g];
                if (o % 128 != 0 || o < prev || o > p.K) { bad = true; o = prev; }
                cum[g] = o;
                prev = o;
            }
            if (bad && rank == 0) record_error(MXFP4_ERR_INVALID_ARG);
            sh->ntiles = p.num_groups * (int)((p.M + 255) / 256) * tiles_n;
        }
    } else {
        if (threadIdx.x == 0) sh->ntiles = (int)((p.M + 255) / 256) * tiles_n;
    }
    // barriers of both CTAs initialized before any cross-CTA traffic
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    const int ntiles = sh->ntiles;
    bool aborted_any = false;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        // The whole warp runs the loop; one elected lane issues the copies.
        const bool issuer = elect_one();
        {
            uint32_t armed = 0, armed_par = 0;   // even CTA: stages armed, parity of the last arm
            int s = 0;
            uint32_t ph = 0;
            for (int t = pair; t < ntiles && !sh->abort; t += npairs) {
                const TileInfo ti = get_tile<BN, MODE>(t, rank, p, cum, tiles_n);
                const int32_t sfa_rt = (int32_t)(ti.row0 / 128);
                const int32_t sfb_rt = (int32_t)(ti.sfb_rt_base + ti.n0 / 128);
                const int ktiles = ktiles_of(ti);
                const int32_t katom0 = (int32_t)(ti.k0 / Cfg::KATOM);   // grouped K: the group's first scale atom
                bool ok = true;
                for (int kt = 0; kt < ktiles; ++kt) {
                    if (!wait_phase(&sh->empty[s], ph ^ 1u, sh, limit)) { ok = false; break; }
                    uint8_t *st = stage_base + s * STAGE_BYTES;
                    const uint32_t full_leader = mapa_shared(smem_u32(&sh->full[s]), 0);
                    if (rank == 0) {
                        armed |= 1u << s;
                        armed_par = (armed_par & ~(1u << s)) | (ph << s);
                    }
                    if (issuer) {
                        if (rank == 0) mbar_arrive_expect_tx(&sh->full[s], Cfg::STAGE_TX);
#pragma unroll
                        for (int c = 0; c < KCH; ++c) {
                            const int32_t kx = (int32_t)(ti.k0 / 2) + (kt * KCH + c) * CHUNK;
                            tma_load_2d_pair(st + c * Cfg::A_CHUNK, &tma_a, kx, (int32_t)ti.row0, full_leader);
                            tma_load_2d_pair(st + A_BYTES + c * Cfg::B_CHUNK, &tma_b, kx,
                                             (int32_t)(ti.b_row + rank * (BN / 2)), full_leader);
                        }
                        // scale atoms: NATOM consecutive K atoms of one (A) or NRT (B) 128-row tiles
                        tma_load_3d_pair(st + A_BYTES + B_BYTES, &tma_sfa, 0, katom0 + kt * NATOM, sfa_rt,
                                         full_leader);
                        tma_load_3d_pair(st + A_BYTES + B_BYTES + SFA_BYTES, &tma_sfb, 0, katom0 + kt * NATOM,
                                         sfb_rt, full_leader);
                    }
                    __syncwarp();
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
            }
            if (rank == 0) {
                // drain: the last load of every armed stage (both CTAs' bytes) has landed
                bool drained = true;
                for (int i = 0; i < STAGES; ++i)
                    if (armed & (1u << i))
                        drained &= wait_phase(&sh->full[i], (armed_par >> i) & 1u, sh, limit, true);
                if (!drained && issuer) mark_drain_failed(sh, rank);
            }
            if (sh->abort) aborted_any = true;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        // The whole warp runs the loop (warp-uniform operands); one elected
        // lane issues each tcgen05 instruction.
        if (rank == 0) {
            bool issued = false;
            int s = 0;
            uint32_t ph = 0, kglobal = 0;
            int acc = 0;
            uint32_t acc_ph = 0;
            for (int t = pair; t < ntiles && !sh->abort; t += npairs) {
                const TileInfo ti = get_tile<BN, MODE>(t, 0, p, cum, tiles_n);
                const int64_t rt0 = ti.n0 / 128;
                const uint32_t b_shift = (uint32_t)((ti.n0 - rt0 * 128) / 32);
                if (!wait_phase(&sh->tmem_empty[acc], acc_ph ^ 1u, sh, limit)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (acc ? Cfg::ACC1_COL : 0u);
                const int ktiles = ktiles_of(ti);
                bool ok = true;
                for (int kt = 0; kt < ktiles; ++kt) {
                    if (!wait_phase(&sh->full[s], ph, sh, limit)) { ok = false; break; }
                    tc_fence_after();
                    const int64_t kleft = ti.kg - (int64_t)kt * Cfg::KSTEP;
                    const uint32_t sfa_col = tmem + Cfg::SF_COL + Cfg::SF_STAGE_COLS * (kglobal & 1u);
                    const uint32_t st = smem_u32(stage_base + s * STAGE_BYTES);
                    if (kleft >= Cfg::KSTEP)
                        issue_stage<Cfg, NATOM, 4 * KCH>(d_tmem, st, sfa_col, b_shift, kt == 0);
                    else
                        issue_stage_tail<Cfg>(d_tmem, st, sfa_col, b_shift, kt == 0, (int)(kleft / 64));
                    issued = true;
                    tc_commit_pair_elect(&sh->empty[s]);
                    ++kglobal;
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit_pair_elect(&sh->tmem_full[acc]);
                if (++acc == 2) { acc = 0; acc_ph ^= 1u; }
            }
            if (issued) {
                // drain: all MMAs / copies of this thread complete before TMEM or smem go away
                tc_commit_pair_elect(&sh->drain);
                if (!wait_phase(&sh->drain, 0, sh, limit, true) && lane == 0) mark_drain_failed(sh, rank);
            }
            if (sh->abort) aborted_any = true;
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int ew = warp - 2;                // epilogue warp index
        const uint32_t empty_leader0 = mapa_shared(smem_u32(&sh->tmem_empty[0]), 0);
        const uint32_t empty_leader1 = mapa_shared(smem_u32(&sh->tmem_empty[1]), 0);
        int acc = 0;
        uint32_t acc_ph = 0;
        uint32_t buf_i = 0;
        // NVFP4: the product of the two second-level scales (amax / 2688 each)
        float nv_scale = 1.0f;
        if constexpr (Cfg::NV) nv_scale = __fmul_rn(__fdiv_rn(*p.a_amax, 2688.0f), __fdiv_rn(*p.b_amax, 2688.0f));
        for (int t = pair; t < ntiles; t += npairs) {
            const TileInfo ti = get_tile<BN, MODE>(t, rank, p, cum, tiles_n);
            if (!wait_phase(&sh->tmem_full[acc], acc_ph, sh, limit)) break;
            tc_fence_after();
            const int row_lo = 32 * q;
            const bool full_box = MODE == MODE_DENSE || (row_lo + 32 <= ti.rows_valid);
            const bool any_row = row_lo < ti.rows_valid;
            const bool empty_k = ti.kg <= 0;              // grouped K: an empty group's output is zero
            if constexpr (OUT == OUT_MX) {
                // fused requantization: after each 32-column TMEM load a lane
                // holds 32 consecutive results of one row, i.e. one 1D row
                // block of C: amax, E8M0 scale and RNE E2M1 codes as in
                // mxfp4_quantize, stored straight from registers
                static_assert(MODE == MODE_DENSE, "MXFP4 output: dense GEMM only");
                const uint32_t tm = tmem + ((uint32_t)(32 * q) << 16) + (acc ? Cfg::ACC1_COL : 0u);
                const int64_t row = ti.c_row0 + row_lo + lane;
                const bool row_ok = row < p.M;
                for (int j = 0; j < BN / 32; ++j) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tm + 32u * j, v);
                    tmem_ld_wait();
                    if (j == BN / 32 - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(acc ? empty_leader1 : empty_leader0);
                    }
                    const int64_t col0 = ti.n0 + 32 * j;
                    if (!row_ok || col0 >= p.N) continue;
                    float f[32];
                    float amax = 0.0f;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        f[i] = __uint_as_float(v[i]);
                        if constexpr (Cfg::NV) f[i] = __fmul_rn(f[i], nv_scale);
                        amax = amax_nan(amax, f[i]);
                    }
                    const uint32_t code = scale_code_from_amax(amax);
                    uint4 qv = make_uint4(0, 0, 0, 0);
                    if (code != 0xFFu) {
                        const float inv = inv_scale_from_code(code);
#pragma unroll
                        for (int i = 0; i < 32; ++i) f[i] = __fmul_rn(f[i], inv);
                        qv = make_uint4(e2m1x8_rn(f), e2m1x8_rn(f + 8), e2m1x8_rn(f + 16), e2m1x8_rn(f + 24));
                    }
                    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(static_cast<uint8_t *>(p.c) +
                                                                                 row * p.ldc + (col0 >> 1)),
                                 "r"(qv.x), "r"(qv.y), "r"(qv.z), "r"(qv.w)
                                 : "memory");
                    const int64_t kb = col0 >> 5;
                    if (p.c_scale_mma) p.c_scales[mma_scale_off(row, kb, p.c_katoms)] = (uint8_t)code;
                    else p.c_scales[row * p.ld_c_scales + kb] = (uint8_t)code;
                }
            } else if constexpr (OUT == OUT_BF16) {
                // 64 columns per step: two 32-column TMEM loads rounded to
                // bf16 pairs (RNE), one 128-byte row segment per lane
                const uint32_t tm = tmem + ((uint32_t)(32 * q) << 16) + (acc ? Cfg::ACC1_COL : 0u);
                for (int j = 0; j < BN / 64; ++j) {
                    uint32_t w[32];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(tm + 64u * j + 32u * h, v);
                        tmem_ld_wait();
                        if (empty_k) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] = 0u;
                        }
                        if constexpr (Cfg::NV) {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                v[i] = __float_as_uint(__fmul_rn(__uint_as_float(v[i]), nv_scale));
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            w[16 * h + i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                    }
                    if (j == BN / 64 - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(acc ? empty_leader1 : empty_leader0);
                    }
                    if (!any_row) continue;
                    const int64_t col0 = ti.n0 + 64 * j;
                    if (col0 >= p.N) continue;
                    if (full_box) {
                        uint8_t *buf = epi_base + (ew * 2 + (buf_i & 1u)) * EPI_BUF;
                        if (lane == 0) bulk_wait_group_read<1>();
                        __syncwarp();
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const uint32_t off = (uint32_t)lane * 128u + (((uint32_t)c ^ (uint32_t)(lane & 7)) << 4);
                            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(buf) + off),
                                         "r"(w[4 * c]), "r"(w[4 * c + 1]), "r"(w[4 * c + 2]), "r"(w[4 * c + 3])
                                         : "memory");
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tma_c, (int32_t)col0, (int32_t)(ti.c_row0 + row_lo), buf);
                            bulk_commit_group();
                        }
                        ++buf_i;
                    } else if (row_lo + lane < ti.rows_valid) {
                        uint16_t *dst = static_cast<uint16_t *>(p.c) + (ti.c_row0 + row_lo + lane) * p.ldc + col0;
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const int64_t cc = col0 + 8 * c;
                            if (cc + 8 <= p.N) {
                                asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(dst + 8 * c),
                                             "r"(w[4 * c]), "r"(w[4 * c + 1]), "r"(w[4 * c + 2]), "r"(w[4 * c + 3])
                                             : "memory");
                            } else {
                                for (int e = 0; e < 8; ++e)
                                    if (cc + e < p.N) dst[8 * c + e] = (uint16_t)(w[4 * c + e / 2] >> (16 * (e & 1)));
                            }
                        }
                    }
                }
            } else {
                for (int j = 0; j < BN / 32; ++j) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (acc ? Cfg::ACC1_COL : 0u) + 32u * j, v);
                    tmem_ld_wait();
                    if (empty_k) {
    #pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = 0u;
                    }
                    if constexpr (Cfg::NV) {
    #pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__fmul_rn(__uint_as_float(v[i]), nv_scale));
                    }
                    if (j == BN / 32 - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(acc ? empty_leader1 : empty_leader0);
                    }
                    if (!any_row) continue;
                    const int64_t col0 = ti.n0 + 32 * j;
                    if (col0 >= p.N) continue;
                    if (full_box) {
                        uint8_t *buf = epi_base + (ew * 2 + (buf_i & 1u)) * EPI_BUF;
                        if (lane == 0) bulk_wait_group_read<1>();
                        __syncwarp();
    #pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const uint32_t off = (uint32_t)lane * 128u + (((uint32_t)c ^ (uint32_t)(lane & 7)) << 4);
                            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(buf) + off),
                                         "r"(v[4 * c]), "r"(v[4 * c + 1]), "r"(v[4 * c + 2]), "r"(v[4 * c + 3])
                                         : "memory");
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tma_c, (int32_t)col0, (int32_t)(ti.c_row0 + row_lo), buf);
                            bulk_commit_group();
                        }
                        ++buf_i;
                    } else if (row_lo + lane < ti.rows_valid) {
                        float *dst = static_cast<float *>(p.c) + (ti.c_row0 + row_lo + lane) * p.ldc + col0;
    #pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const int64_t cc = col0 + 4 * c;
                            if (cc + 4 <= p.N) {
                                asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(dst + 4 * c), "r"(v[4 * c]),
                                             "r"(v[4 * c + 1]), "r"(v[4 * c + 2]), "r"(v[4 * c + 3])
                                             : "memory");
                            } else {
                                for (int e = 0; e < 4; ++e)
                                    if (cc + e < p.N) dst[4 * c + e] = __uint_as_float(v[4 * c + e]);
                            }
                        }
                    }
                }
            }
            if (++acc == 2) { acc = 0; acc_ph ^= 1u; }
        }
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
        if (sh->abort) aborted_any = true;
    }
    (void)aborted_any;
    __syncthreads();
    cluster_sync();   // neither CTA leaves while the pair may still touch its smem or TMEM
    // The leader's drain waited (bounded) for every load of both CTAs and for
    // its MMAs; only if such a wait ran out can a copy or an MMA still be in
    // flight: then give it time before the shared and tensor memory go away.
    if (sh->drain_failed) spin_ns(200000);
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

// Bounded-wait probe: one barrier that only `arrive` can complete.
__global__ void wait_probe_kernel(int arrive, uint64_t limit) {
    __shared__ uint64_t bar;
    __shared__ Shared sh;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        sh.abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (arrive) mbar_arrive(&bar);
        wait_phase(&bar, 0, &sh, limit);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static uint64_t g_wait_limit_ns = 2000000000ull;

uint64_t set_wait_limit(uint64_t ns) {
    const uint64_t old = g_wait_limit_ns;
    g_wait_limit_ns = ns ? ns : 2000000000ull;
    return old;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

static bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                     uint64_t stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scale atoms of the GEMM-ready layout: 512-byte atoms, katoms per 128-row
// tile, `tiles` row tiles; boxes of `box_k` atoms x `box_t` tiles.
static bool make_map_3d(CUtensorMap *m, const void *base, uint64_t katoms, uint64_t tiles, uint32_t box_k,
                        uint32_t box_t) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {128, katoms, tiles};
    const cuuint64_t strides[2] = {512, 512 * katoms};
    const cuuint32_t box[3] = {128, box_k, box_t};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int sm_count() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

template <class Cfg, int MODE, int OUT>
static cudaError_t set_smem_attr() {
    // once per device and instantiation: keep cudaFuncSetAttribute off the hot path
    static int done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(mxfp4_gemm_kernel<Cfg, MODE, OUT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = 1;
    return e;
}

struct GemmArgs {
    const uint8_t *a_codes, *a_scales, *b_codes, *b_scales;
    int64_t lda, ldb, M, N, K, ldc;
    void *c;
    const int32_t *offsets, *sizes;
    int G;
    const float *a_amax = nullptr, *b_amax = nullptr;
    uint8_t *c_scales = nullptr;
    int64_t ld_c_scales = 0;
    int c_scale_mma = 0;
};

// Returns 0 on success, MXFP4_ERR_CUDA when a map or launch fails.
// Grouped K: a and b are [M, K/2] and [N, K/2] over all groups' K ranges, c is
// [G * M, N]; the B operand and C map cover G groups only in grouped-rows mode.
// OUT_BF16: C is bf16 (RNE of the FP32 accumulators), stored in 64-column
// boxes; OUT_MX: C is MXFP4 codes + scales written without the C tensor map
// (a map over the codes is still passed, never used).
template <class Cfg, int MODE, int OUT = OUT_F32>
static int launch_cfg(const GemmArgs &g, cudaStream_t s) {
    constexpr int BN = Cfg::BN;
    const int G = MODE == MODE_GROUPED_M ? g.G : 1;
    const int64_t c_rows = MODE == MODE_GROUPED_K ? (int64_t)g.G * g.M : g.M;
    const int64_t katoms = (g.K + Cfg::KATOM - 1) / Cfg::KATOM;
    const int64_t a_tiles = (g.M + 127) / 128, b_tiles = (g.N + 127) / 128;
    CUtensorMap ta, tb, tc, tsa, tsb;
    if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a_codes, (uint64_t)(g.K / 2), (uint64_t)g.M,
                  (uint64_t)g.lda, CHUNK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.b_codes, (uint64_t)(g.K / 2), (uint64_t)G * g.N,
                  (uint64_t)g.ldb, CHUNK, BN / 2, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !(OUT == OUT_MX
              ? make_map(&tc, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.c, (uint64_t)(g.N / 2), (uint64_t)c_rows,
                         (uint64_t)g.ldc, 16, 32, CU_TENSOR_MAP_SWIZZLE_NONE)
              : make_map(&tc, OUT == OUT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                         g.c, (uint64_t)g.N, (uint64_t)c_rows, (uint64_t)g.ldc * (OUT == OUT_BF16 ? 2 : 4),
                         OUT == OUT_BF16 ? 64 : 32, 32, CU_TENSOR_MAP_SWIZZLE_128B)) ||
        // scale atoms as a 3D tensor [128-row tile][K atom][512 bytes = 128 x 32-bit]:
        // one box holds NATOM consecutive atoms of one (A) or NRT (B) row tiles
        !make_map_3d(&tsa, g.a_scales, (uint64_t)katoms, (uint64_t)a_tiles, Cfg::NATOM, 1) ||
        !make_map_3d(&tsb, g.b_scales, (uint64_t)katoms, (uint64_t)(G * b_tiles), Cfg::NATOM, Cfg::NRT))
        return MXFP4_ERR_CUDA;
    if (set_smem_attr<Cfg, MODE, OUT>() != cudaSuccess) return MXFP4_ERR_CUDA;
    GemmParams p{};
    p.M = g.M; p.N = g.N; p.K = g.K;
    p.katoms = katoms;
    p.b_rowtiles = b_tiles;
    p.c = g.c; p.ldc = g.ldc;
    p.c_scales = g.c_scales; p.ld_c_scales = g.ld_c_scales; p.c_scale_mma = g.c_scale_mma;
    p.c_katoms = (g.N / 32 + 3) / 4;
    p.group_offsets = g.offsets; p.group_sizes = g.sizes; p.num_groups = g.G;
    p.a_amax = g.a_amax; p.b_amax = g.b_amax;
    p.wait_limit_ns = g_wait_limit_ns;
    const int pairs_max = sm_count() / 2;
    int pairs = pairs_max;
    if (MODE != MODE_GROUPED_M) {
        const int64_t tiles = (MODE == MODE_GROUPED_K ? g.G : 1) * ((g.M + 255) / 256) * ((g.N + BN - 1) / BN);
        pairs = (int)(tiles < pairs_max ? tiles : pairs_max);
    }
    const cudaError_t e = launch_pdl(mxfp4_gemm_kernel<Cfg, MODE, OUT>, dim3((unsigned)(2 * pairs)), dim3(NUM_THREADS),
                                     (size_t)Cfg::SMEM_BYTES, s, ta, tb, tc, tsa, tsb, p);
    return e == cudaSuccess ? 0 : MXFP4_ERR_CUDA;
}

int launch_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes, int64_t ldb,
                const uint8_t *b_scales, int64_t M, int64_t N, int64_t K, float *c, int64_t ldc, cudaStream_t s) {
    GemmArgs g{a_codes, a_scales, b_codes, b_scales, lda, ldb, M, N, K, ldc, c, nullptr, nullptr, 1};
    return launch_cfg<DefaultCfg, MODE_DENSE>(g, s);
}

int launch_grouped_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, int64_t a_rows,
                        const int32_t *offsets, const int32_t *sizes, int G, const uint8_t *b_codes, int64_t ldb,
                        const uint8_t *b_scales, int64_t N, int64_t K, float *c, int64_t ldc, cudaStream_t s) {
    GemmArgs g{a_codes, a_scales, b_codes, b_scales, lda, ldb, a_rows, N, K, ldc, c, offsets, sizes, G};
    return launch_cfg<DefaultCfg, MODE_GROUPED_M>(g, s);
}

int launch_gemm_bf16(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes,
                     int64_t ldb, const uint8_t *b_scales, int64_t M, int64_t N, int64_t K, uint16_t *c, int64_t ldc,
                     cudaStream_t s) {
    GemmArgs g{a_codes, a_scales, b_codes, b_scales, lda, ldb, M, N, K, ldc, c, nullptr, nullptr, 1};
    return launch_cfg<DefaultCfg, MODE_DENSE, OUT_BF16>(g, s);
}

int launch_grouped_gemm_bf16(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, int64_t a_rows,
                             const int32_t *offsets, const int32_t *sizes, int G, const uint8_t *b_codes,
                             int64_t ldb, const uint8_t *b_scales, int64_t N, int64_t K, uint16_t *c, int64_t ldc,
                             cudaStream_t s) {
    GemmArgs g{a_codes, a_scales, b_codes, b_scales, lda, ldb, a_rows, N, K, ldc, c, offsets, sizes, G};
    return launch_cfg<DefaultCfg, MODE_GROUPED_M, OUT_BF16>(g, s);
}

int launch_gemm_mx(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes,
                   int64_t ldb, const uint8_t *b_scales, int64_t M, int64_t N, int64_t K, uint8_t *c_codes,
                   int64_t ld_c_codes, uint8_t *c_scales, int64_t ld_c_scales, int c_scale_mma, cudaStream_t s) {
    GemmArgs g{a_codes, a_scales, b_codes, b_scales, lda, ldb, M, N, K, ld_c_codes, c_codes, nullptr, nullptr, 1};
    g.c_scales = c_scales;
    g.ld_c_scales = ld_c_scales;
    g.c_scale_mma = c_scale_mma;
    return launch_cfg<DefaultCfg, MODE_DENSE, OUT_MX>(g, s);
}

int launch_grouped_wgrad(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes,
                         int64_t ldb, const uint8_t *b_scales, const int32_t *offsets, int G, int64_t M, int64_t N,
                         int64_t K, float *c, int64_t ldc, cudaStream_t s) {
    GemmArgs g{a_codes, a_scales, b_codes, b_scales, lda, ldb, M, N, K, ldc, c, offsets, nullptr, G};
    return launch_cfg<DefaultCfg, MODE_GROUPED_K>(g, s);
}

int launch_grouped_wgrad_bf16(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes,
                              int64_t ldb, const uint8_t *b_scales, const int32_t *offsets, int G, int64_t M,
                              int64_t N, int64_t K, uint16_t *c, int64_t ldc, cudaStream_t s) {
    GemmArgs g{a_codes, a_scales, b_codes, b_scales, lda, ldb, M, N, K, ldc, c, offsets, nullptr, G};
    return launch_cfg<DefaultCfg, MODE_GROUPED_K, OUT_BF16>(g, s);
}

int launch_nvfp4_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const float *a_amax,
                      const uint8_t *b_codes, int64_t ldb, const uint8_t *b_scales, const float *b_amax, int64_t M,
                      int64_t N, int64_t K, float *c, int64_t ldc, cudaStream_t s) {
    GemmArgs g{a_codes, a_scales, b_codes, b_scales, lda, ldb, M, N, K, ldc, c, nullptr, nullptr, 1, a_amax, b_amax};
    return launch_cfg<NvCfg, MODE_DENSE>(g, s);
}

int get_error(cudaStream_t s) {
    if (cudaStreamSynchronize(s) != cudaSuccess) return MXFP4_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_error_code, sizeof(v)) != cudaSuccess) return MXFP4_ERR_CUDA;
    const unsigned int zero = 0;
    if (v && cudaMemcpyToSymbol(g_error_code, &zero, sizeof(zero)) != cudaSuccess) return MXFP4_ERR_CUDA;
    return (int)v;
}

int launch_wait_probe(int arrive, cudaStream_t s) {
    wait_probe_kernel<<<1, 32, 0, s>>>(arrive, g_wait_limit_ns);
    return cudaGetLastError() == cudaSuccess ? 0 : MXFP4_ERR_CUDA;
}

}  // namespace mxfp4
