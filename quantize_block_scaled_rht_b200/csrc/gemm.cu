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
// Kernel structure (persistent, one CTA per SM, 6 warps):
//   warp 0      TMA producer: A/B code tiles (128x256 and 192x256 E2M1,
//               128-byte swizzle) and the matching scale atoms (bulk copies of
//               the GEMM-ready scale layout) into a 4-stage shared-memory ring;
//   warp 1      MMA issuer: copies the stage's scale atoms to TMEM
//               (tcgen05.cp 32x128b.warpx4), issues 4 MMAs per stage into one
//               of two TMEM accumulators (128 x 192 FP32 each), releases the
//               stage with tcgen05.commit;
//   warps 2..5  epilogue: TMEM -> registers (tcgen05.ld) -> swizzled smem ->
//               TMA store of FP32 C, overlapping the next tile's MMAs.
// Every barrier wait is bounded by the GPU global timer; a wait that runs out
// records MXFP4_ERR_TIMEOUT, raises a CTA-wide abort flag and every role
// drains its own in-flight copies / MMAs before the CTA exits.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mxfp4 {

constexpr int BM = 128, BN = 192, BKB = 128;          // tile rows, tile cols, K bytes per stage (256 E2M1)
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BKB;                     // 16 KB
constexpr int B_BYTES = BN * BKB;                     // 24 KB
constexpr int SFA_BYTES = 2 * 512;                    // 2 K-atoms of 128 rows
constexpr int SFB_BYTES = 2 * 2 * 512;                // 2 row tiles x 2 K-atoms
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;   // 44032 = 43 KB
constexpr int EPI_WARPS = 4;
constexpr int EPI_BUF = 32 * 32 * 4;                  // 32 rows x 32 FP32
constexpr int EPI_BYTES = EPI_WARPS * 2 * EPI_BUF;
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_STRIDE = 256;                  // accumulator b at column 256 b
constexpr uint32_t SF_COL = 192;                      // scale factors: [192, 240)
constexpr int MAX_GROUPS = 1024;

// Instruction descriptor, kind::mxf4 block-scaled: A/B E2M1 (1), K-major,
// N >> 3 at bit 17, UE8M0 scales (bit 23), M >> 4 at bit 24, scale-factor
// byte selectors at bits 4 (B) and 29 (A).
constexpr uint32_t IDESC_BASE = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | (1u << 23) |
                                ((uint32_t)(BM >> 4) << 24);

__device__ unsigned int g_error_code;

__device__ __forceinline__ void record_error(unsigned int code) { atomicCAS(&g_error_code, 0u, code); }

struct GemmParams {
    const uint8_t *a_scales;
    const uint8_t *b_scales;
    int64_t M, N, K;
    int64_t katoms;            // ceil(K / 128): scale atoms per 128-row tile
    int64_t b_rowtiles;        // ceil(N / 128)
    int64_t b_group_sf_bytes;  // grouped: MMA scale bytes of one expert
    float *c;
    int64_t ldc;
    const int32_t *group_offsets;
    const int32_t *group_sizes;
    int num_groups;
    uint64_t wait_limit_ns;
};

struct Shared {
    uint64_t full[STAGES], empty[STAGES];
    uint64_t tmem_full[2], tmem_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    volatile int abort;
    int ntiles;
};

// Bounded wait: true once the phase of `parity` has completed; false if the
// CTA aborted or the wait ran past the limit (which records the timeout and
// aborts the CTA).  `hard` waits ignore the abort flag (used while draining).
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, Shared *sh, uint64_t limit, bool hard = false) {
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

struct TileInfo {
    int64_t row0;       // first A/C row
    int rows_valid;     // rows of this tile that belong to the problem (grouped: to the group)
    int64_t n0;         // first C column
    int64_t b_row;      // TMA row coordinate of the first B row
    const uint8_t *sfb; // scale base of this B operand (expert)
};

template <bool GROUPED>
__device__ __forceinline__ TileInfo get_tile(int t, const GemmParams &p, const int *cum, int tiles_n) {
    TileInfo ti;
    if constexpr (!GROUPED) {
        const int tiles_m = (int)((p.M + BM - 1) / BM);
        const int tm = t % tiles_m, tn = t / tiles_m;
        ti.row0 = (int64_t)tm * BM;
        const int64_t left = p.M - ti.row0;
        ti.rows_valid = left < BM ? (int)left : BM;
        ti.n0 = (int64_t)tn * BN;
        ti.b_row = ti.n0;
        ti.sfb = p.b_scales;
    } else {
        int g = 0;
        while (g + 1 < p.num_groups && cum[g + 1] <= t) ++g;
        const int local = t - cum[g];
        const int tiles_g = (cum[g + 1] - cum[g]) / tiles_n;
        const int tm = local % tiles_g, tn = local / tiles_g;
        const int64_t size = p.group_sizes[g];
        ti.row0 = (int64_t)p.group_offsets[g] + (int64_t)tm * BM;
        const int64_t left = size - (int64_t)tm * BM;
        ti.rows_valid = left < BM ? (int)left : BM;
        ti.n0 = (int64_t)tn * BN;
        ti.b_row = (int64_t)g * p.N + ti.n0;
        ti.sfb = p.b_scales + (int64_t)g * p.b_group_sf_bytes;
    }
    return ti;
}

template <bool GROUPED>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    mxfp4_gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                      const __grid_constant__ CUtensorMap tma_c, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *stage_base = smem;
    uint8_t *epi_base = smem + STAGES * STAGE_BYTES;
    Shared *sh = reinterpret_cast<Shared *>(epi_base + EPI_BYTES);
    __shared__ int cum[GROUPED ? MAX_GROUPS + 1 : 1];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_n = (int)((p.N + BN - 1) / BN);
    const int ktiles = (int)((p.K / 2 + BKB - 1) / BKB);
    const uint64_t limit = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(&sh->full[s], 1); mbar_init(&sh->empty[s], 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(&sh->tmem_full[b], 1); mbar_init(&sh->tmem_empty[b], EPI_WARPS); }
        mbar_init(&sh->drain, 1);
        sh->abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
        prefetch_tmap(&tma_a);
        prefetch_tmap(&tma_b);
        prefetch_tmap(&tma_c);
    }
    if (warp == 1) {
        tmem_alloc(&sh->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    if constexpr (GROUPED) {
        if (threadIdx.x == 32 * 2) {
            int acc = 0;
            for (int g = 0; g < p.num_groups; ++g) {
                cum[g] = acc;
                const int64_t off = p.group_offsets[g], nxt = p.group_offsets[g + 1];
                int64_t size = p.group_sizes[g];
                int tm = 0;
                if ((off % BM) != 0 || size < 0 || off + size > nxt) {
                    record_error(MXFP4_ERR_INVALID_ARG);
                } else {
                    tm = (int)((size + BM - 1) / BM);
                }
                acc += tm * tiles_n;
            }
            cum[p.num_groups] = acc;
            sh->ntiles = acc;
        }
    } else {
        if (threadIdx.x == 0) sh->ntiles = (int)((p.M + BM - 1) / BM) * tiles_n;
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    const int ntiles = sh->ntiles;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t armed = 0, armed_par = 0;   // per stage: armed at least once, parity of last arm
            int s = 0;
            uint32_t ph = 0;
            for (int t = blockIdx.x; t < ntiles && !sh->abort; t += gridDim.x) {
                const TileInfo ti = get_tile<GROUPED>(t, p, cum, tiles_n);
                const int64_t rt0 = ti.n0 / 128;
                const int nrt = (rt0 + 1 < p.b_rowtiles) ? 2 : 1;
                const uint8_t *sfa_src = p.a_scales + ((ti.row0 / 128) * p.katoms) * 512;
                bool ok = true;
                for (int kt = 0; kt < ktiles; ++kt) {
                    if (!wait_phase(&sh->empty[s], ph ^ 1u, sh, limit)) { ok = false; break; }
                    const int natoms = (int)((p.katoms - 2 * kt) < 2 ? (p.katoms - 2 * kt) : 2);
                    const uint32_t sf_bytes = (uint32_t)natoms * 512u;
                    uint8_t *st = stage_base + s * STAGE_BYTES;
                    mbar_arrive_expect_tx(&sh->full[s], A_BYTES + B_BYTES + sf_bytes * (1 + nrt));
                    tma_load_2d(st, &tma_a, kt * BKB, (int32_t)ti.row0, &sh->full[s]);
                    tma_load_2d(st + A_BYTES, &tma_b, kt * BKB, (int32_t)ti.b_row, &sh->full[s]);
                    bulk_load(st + A_BYTES + B_BYTES, sfa_src + (int64_t)(2 * kt) * 512, sf_bytes, &sh->full[s]);
                    for (int rt = 0; rt < nrt; ++rt)
                        bulk_load(st + A_BYTES + B_BYTES + SFA_BYTES + rt * 1024,
                                  ti.sfb + ((rt0 + rt) * p.katoms + 2 * kt) * 512, sf_bytes, &sh->full[s]);
                    armed |= 1u << s;
                    armed_par = (armed_par & ~(1u << s)) | (ph << s);
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
            }
            // drain: every armed stage's last load must have landed before exit
            for (int i = 0; i < STAGES; ++i)
                if (armed & (1u << i)) wait_phase(&sh->full[i], (armed_par >> i) & 1u, sh, limit, true);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool issued = false;
            int s = 0;
            uint32_t ph = 0, kglobal = 0;
            int acc = 0;
            uint32_t acc_ph = 0;
            for (int t = blockIdx.x; t < ntiles && !sh->abort; t += gridDim.x) {
                const TileInfo ti = get_tile<GROUPED>(t, p, cum, tiles_n);
                const int64_t rt0 = ti.n0 / 128;
                const int nrt = (rt0 + 1 < p.b_rowtiles) ? 2 : 1;
                const uint32_t b_shift = (uint32_t)((ti.n0 - rt0 * 128) / 32);
                if (!wait_phase(&sh->tmem_empty[acc], acc_ph ^ 1u, sh, limit)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)acc * ACC_STRIDE;
                bool ok = true;
                for (int kt = 0; kt < ktiles; ++kt) {
                    if (!wait_phase(&sh->full[s], ph, sh, limit)) { ok = false; break; }
                    tc_fence_after();
                    const int natoms = (int)((p.katoms - 2 * kt) < 2 ? (p.katoms - 2 * kt) : 2);
                    const int64_t kleft = p.K - (int64_t)kt * 256;
                    const int nk = kleft >= 256 ? 4 : (int)(kleft / 64);
                    const uint32_t sfa_col = SF_COL + 24u * (kglobal & 1u);
                    const uint32_t sfb_col = sfa_col + 8u;
                    const uint32_t st = smem_u32(stage_base + s * STAGE_BYTES);
                    const uint32_t sfa_s = st + A_BYTES + B_BYTES, sfb_s = sfa_s + SFA_BYTES;
                    for (int a = 0; a < natoms; ++a) {
                        tc_cp_32x128_warpx4(tmem + sfa_col + 4u * a, smem_desc(sfa_s + 512u * a, 0, 128, 0));
                        for (int rt = 0; rt < nrt; ++rt)
                            tc_cp_32x128_warpx4(tmem + sfb_col + 8u * a + 4u * rt,
                                                smem_desc(sfb_s + 1024u * rt + 512u * a, 0, 128, 0));
                    }
                    const uint64_t adesc = smem_desc(st, 16, 1024, 2);
                    const uint64_t bdesc = smem_desc(st + A_BYTES, 16, 1024, 2);
                    for (int k = 0; k < nk; ++k) {
                        const uint32_t sel = 2u * (uint32_t)(k & 1);
                        const uint32_t idesc = IDESC_BASE | (sel << 29) | (sel << 4);
                        mma_mxf4(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), idesc,
                                 tmem + sfa_col + 4u * (uint32_t)(k >> 1),
                                 tmem + sfb_col + 8u * (uint32_t)(k >> 1) + b_shift, (kt | k) != 0);
                    }
                    issued = true;
                    tc_commit(&sh->empty[s]);
                    ++kglobal;
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&sh->tmem_full[acc]);
                if (++acc == 2) { acc = 0; acc_ph ^= 1u; }
            }
            if (issued) {
                // drain: all MMAs / copies of this thread complete before TMEM is freed
                tc_commit(&sh->drain);
                wait_phase(&sh->drain, 0, sh, limit, true);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int ew = warp - 2;                // epilogue warp index
        int acc = 0;
        uint32_t acc_ph = 0;
        uint32_t buf_i = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            const TileInfo ti = get_tile<GROUPED>(t, p, cum, tiles_n);
            if (!wait_phase(&sh->tmem_full[acc], acc_ph, sh, limit)) break;
            tc_fence_after();
            const int row_lo = 32 * q;
            const bool full_box = !GROUPED || (row_lo + 32 <= ti.rows_valid);
            const bool any_row = row_lo < ti.rows_valid;
            for (int j = 0; j < BN / 32; ++j) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)acc * ACC_STRIDE + 32u * j, v);
                tmem_ld_wait();
                if (j == BN / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh->tmem_empty[acc]);
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
                        tma_store_2d(&tma_c, (int32_t)col0, (int32_t)(ti.row0 + row_lo), buf);
                        bulk_commit_group();
                    }
                    ++buf_i;
                } else if (row_lo + lane < ti.rows_valid) {
                    float *dst = p.c + (ti.row0 + row_lo + lane) * p.ldc + col0;
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
            if (++acc == 2) { acc = 0; acc_ph ^= 1u; }
        }
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
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
                     uint64_t stride_bytes, uint32_t box_inner, uint32_t box_outer) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int sm_count() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

template <bool GROUPED>
static cudaError_t set_smem_attr() {
    // per device: cudaFuncSetAttribute is cheap, but keep it off the hot path
    static int done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(mxfp4_gemm_kernel<GROUPED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM_BYTES);
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = 1;
    return e;
}

// Returns 0 on success, MXFP4_ERR_CUDA when a map or launch fails.
int launch_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, const uint8_t *b_codes, int64_t ldb,
                const uint8_t *b_scales, int64_t M, int64_t N, int64_t K, float *c, int64_t ldc, cudaStream_t s) {
    CUtensorMap ta, tb, tc;
    if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, (uint64_t)(K / 2), (uint64_t)M, (uint64_t)lda, BKB, BM) ||
        !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, b_codes, (uint64_t)(K / 2), (uint64_t)N, (uint64_t)ldb, BKB, BN) ||
        !make_map(&tc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, c, (uint64_t)N, (uint64_t)M, (uint64_t)ldc * 4, 32, 32))
        return MXFP4_ERR_CUDA;
    if (set_smem_attr<false>() != cudaSuccess) return MXFP4_ERR_CUDA;
    GemmParams p{};
    p.a_scales = a_scales; p.b_scales = b_scales;
    p.M = M; p.N = N; p.K = K;
    p.katoms = mma_katoms(K);
    p.b_rowtiles = (N + 127) / 128;
    p.c = c; p.ldc = ldc;
    p.wait_limit_ns = g_wait_limit_ns;
    const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int sms = sm_count();
    const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
    mxfp4_gemm_kernel<false><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(ta, tb, tc, p);
    return cudaGetLastError() == cudaSuccess ? 0 : MXFP4_ERR_CUDA;
}

int launch_grouped_gemm(const uint8_t *a_codes, int64_t lda, const uint8_t *a_scales, int64_t a_rows,
                        const int32_t *offsets, const int32_t *sizes, int G, const uint8_t *b_codes, int64_t ldb,
                        const uint8_t *b_scales, int64_t N, int64_t K, float *c, int64_t ldc, cudaStream_t s) {
    CUtensorMap ta, tb, tc;
    if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, (uint64_t)(K / 2), (uint64_t)a_rows, (uint64_t)lda, BKB,
                  BM) ||
        !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, b_codes, (uint64_t)(K / 2), (uint64_t)(G * N), (uint64_t)ldb,
                  BKB, BN) ||
        !make_map(&tc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, c, (uint64_t)N, (uint64_t)a_rows, (uint64_t)ldc * 4, 32, 32))
        return MXFP4_ERR_CUDA;
    if (set_smem_attr<true>() != cudaSuccess) return MXFP4_ERR_CUDA;
    GemmParams p{};
    p.a_scales = a_scales; p.b_scales = b_scales;
    p.M = a_rows; p.N = N; p.K = K;
    p.katoms = mma_katoms(K);
    p.b_rowtiles = (N + 127) / 128;
    p.b_group_sf_bytes = ((N + 127) / 128) * p.katoms * 512;
    p.c = c; p.ldc = ldc;
    p.group_offsets = offsets; p.group_sizes = sizes; p.num_groups = G;
    p.wait_limit_ns = g_wait_limit_ns;
    mxfp4_gemm_kernel<true><<<(unsigned)sm_count(), NUM_THREADS, SMEM_BYTES, s>>>(ta, tb, tc, p);
    return cudaGetLastError() == cudaSuccess ? 0 : MXFP4_ERR_CUDA;
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
