// Persistent, warp-specialised FP8 block-scaled GEMM for sm_100a.
//
// D = A . B^T with E4M3 operands, packed UE8M0 scales (one per 1x128 block of
// A, one per 128x128 block of B), fp32 accumulation in TMEM, bf16 output. One
// template serves the three forms of the method ("DeepInside DeepGEMM" section
// 4 for the dense NT GEMM; "DeepGEMM CUDA Graph Compatibility for Masked
// Grouped GEMMs" for the masked form; the contiguous form is the "continuous
// storage layout" of "DeepGEMM tested by Novita AI").
//
// CTA = 6 warps, one CTA per SM, grid fixed by the problem sizes:
//   warp 0      producer: TMA loads of the A and B tiles (128-byte swizzle)
//               into a STAGES-deep shared-memory ring; every 4th K-block it
//               also gathers the packed scale words (one int32 = 4 K-blocks)
//               into the 32x16-byte layout that tcgen05.cp expects.
//   warp 1      MMA issuer: allocates TMEM, copies the scale words to TMEM,
//               issues tcgen05.mma.kind::mxf8f6f4.block_scale (M=128, N=BN,
//               K=32) four times per 128-K block, selecting the UE8M0 byte of
//               the current K-block with the scale-factor id, and commits
//               stage releases and accumulator hand-offs to mbarriers.
//   warps 2..5  epilogue: TMEM -> registers (tcgen05.ld, up to 128 columns
//               per batch; TMEM is handed back right after the last read),
//               fp32 -> bf16 with round-to-nearest-even, 32x32 chunks staged
//               in swizzled shared memory and written by TMA; chunks holding
//               rows that must not be written (past masked_m, padding of
//               m_indices) use predicated row stores instead, so those rows
//               are never touched.
// The accumulator is double-buffered in TMEM when two fit next to the scale
// columns, so the epilogue of tile i overlaps the MMAs of tile i+1.
//
// Block scaling: the hardware MMA applies one UE8M0 scale per 32 K values for
// each row of A and each column of B. The 128-granular scales of this format
// are the same for the four K=32 MMAs of a K-block, so each of them is issued
// with the byte selector (K-block mod 4) into the packed word, i.e. the packed
// int32 words are copied to TMEM as they are, once per four K-blocks.
//
// Every mbarrier wait is bounded; on timeout the kernel records
// DG_DEVERR_TIMEOUT in the device status word and unwinds.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda.h>

#include "ptx.cuh"

namespace dg {

enum GemmKind : int { kDense = 0, kContiguous = 1, kMasked = 2 };

constexpr int BM = 128;                 // rows per tile (one MMA, cta_group::1)
constexpr int BK = 128;                 // K per pipeline stage = one scale block
constexpr int MMA_K = 32;               // K of one kind::mxf8f6f4 MMA
constexpr int NUM_THREADS = 192;
constexpr int MAX_MASKED_GROUPS = 1024;
constexpr int SMEM_LIMIT = 232448;      // 227 KB opt-in per CTA
constexpr uint64_t DEFAULT_WAIT_LIMIT_NS = 2000000000ull;  // 2 s

constexpr uint32_t DEVERR_TIMEOUT = 1u;
constexpr uint32_t DEVERR_MIXED_EXPERT_BLOCK = 2u;

struct GemmParams {
    CUtensorMap tma_a;        // A: 2-D {K, rows} (dense, contiguous) or 3-D {K, max_m, G} (masked)
    CUtensorMap tma_b;        // B: 2-D {K, N} (dense) or 3-D {K, N, G} (grouped)
    CUtensorMap tma_d;        // D (bf16, store): 2-D {N, rows} or 3-D {N, max_m, G}; 32x32 box, 64-byte swizzle
    const int32_t* sfa;       // packed scale rows of A
    const int32_t* sfb;       // packed scale rows of B (per 128 rows, per group)
    __nv_bfloat16* d;         // output
    const int32_t* meta;      // m_indices (contiguous) / masked_m (masked) / null
    uint32_t* status;         // device status word
    int rows;                 // M (dense), M_total (contiguous), max_m (masked)
    int n, k, groups;
    int kb;                   // K / 128
    int kp;                   // ceil(kb / 4) packed words per scale row
    int nb_sf;                // ceil(N / 128) scale rows per weight matrix
    int num_m_blocks;         // ceil(rows / 128)
    int num_n_blocks;         // ceil(N / BN)
    int raster_group;         // m-blocks per raster band (dense / contiguous)
    uint64_t wait_limit_ns;   // bound of every mbarrier wait
    int test_mode;            // 1: CTA 0 withholds one stage arrive (exercises the timeout path)
};

template <int BN>
struct GemmConfig {
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "N tile must be a multiple of 32 in [32, 256]");
    static constexpr int A_BYTES = BM * BK;
    static constexpr int B_BYTES = BN * BK;
    static constexpr int SFB_CHUNKS = (BN + 127) / 128;         // 128-column chunks of B scales
    static constexpr int SFA_BYTES = 512;                       // 32 rows x 16 bytes
    static constexpr int SFB_BYTES = 512 * SFB_CHUNKS;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int EPI_WARP_BYTES = 2 * 2048;                // two 32x32 bf16 staging buffers per warp
    static constexpr int EPI_BYTES = 4 * EPI_WARP_BYTES;
    static constexpr int FIXED_BYTES =
        1024 /*align slack*/ + EPI_BYTES + 512 /*barriers*/ + (2 * MAX_MASKED_GROUPS + 8) * 4;
    static constexpr int STAGES_FIT = (SMEM_LIMIT - FIXED_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
    static_assert(STAGES >= 2, "pipeline too shallow");
    static constexpr int SMEM_BYTES = FIXED_BYTES + STAGES * STAGE_BYTES;

    // TMEM columns: accumulator slot(s), then 4 columns of A scales and
    // 4 per 128-column chunk of B scales.
    static constexpr int ACC_COLS = ((BN + 31) / 32) * 32;
    static constexpr int SF_COLS = 4 + 4 * SFB_CHUNKS;
    static constexpr int NUM_ACC = (2 * ACC_COLS + SF_COLS <= 512) ? 2 : 1;
    static constexpr int SFA_COL = NUM_ACC * ACC_COLS;
    static constexpr int SFB_COL = SFA_COL + 4;
    static_assert(SFB_COL + 4 * SFB_CHUNKS <= 512, "TMEM overflow");
    static constexpr uint32_t TMEM_COLS = 512;
};

struct Tile {
    int m_blk, n_blk, g;      // g: group (masked) or expert (contiguous), 0 for dense
};

// ----------------------------------------------------------------- waits ----

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of `bar` with the given parity. Gives up when another
// role of this CTA has given up, or after p.wait_limit_ns; a timeout is
// recorded in the device status word.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, const GemmParams& p,
                                             volatile int* s_abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*s_abort) return false;
        if (global_ns() - t0 > p.wait_limit_ns) {
            atomicOr(p.status, DEVERR_TIMEOUT);
            *s_abort = 1;
            return false;
        }
    }
}

// Bounded wait used only while unwinding: no status update.
__device__ __forceinline__ void wait_quiet(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity) && global_ns() - t0 < limit_ns) {
    }
}

// ------------------------------------------------------------- scheduling --

// Dense / contiguous: banded raster. Within a band of `raster_group` m-blocks
// the m-block varies fastest, so CTAs running at the same time share the B tile
// and a bounded slab of A.
__device__ __forceinline__ bool raster_tile(const GemmParams& p, int t, Tile& c) {
    const int total = p.num_m_blocks * p.num_n_blocks;
    if (t >= total) return false;
    const int band_tiles = p.raster_group * p.num_n_blocks;
    const int band = t / band_tiles;
    const int local = t - band * band_tiles;
    const int m0 = band * p.raster_group;
    const int gm = min(p.raster_group, p.num_m_blocks - m0);
    c.n_blk = local / gm;
    c.m_blk = m0 + (local - c.n_blk * gm);
    c.g = 0;
    return true;
}

// Masked: tiles of group g are numbered from s_prefix[g]; within a group the
// m-block varies fastest. `gcur` is the caller's monotone cursor.
__device__ __forceinline__ bool masked_tile(const int* s_prefix, const int* s_mm, int groups, int t, int& gcur,
                                            Tile& c) {
    if (t >= s_prefix[groups]) return false;
    while (s_prefix[gcur + 1] <= t) ++gcur;
    const int local = t - s_prefix[gcur];
    const int mb = (s_mm[gcur] + BM - 1) / BM;
    c.g = gcur;
    c.n_blk = local / mb;
    c.m_blk = local - c.n_blk * mb;
    return true;
}

// Contiguous: expert of an aligned 128-row block = largest valid index among
// its rows (-1 if none). Whole warp.
__device__ __forceinline__ int block_expert(const GemmParams& p, int m_blk, uint32_t lane) {
    int best = -1;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int r = m_blk * BM + 32 * j + static_cast<int>(lane);
        if (r < p.rows) {
            const int id = __ldg(p.meta + r);
            if (id >= 0 && id < p.groups) best = max(best, id);
        }
    }
    return __reduce_max_sync(0xffffffffu, best);
}

template <int KIND, bool NEED_EXPERT>
__device__ __forceinline__ bool next_tile(const GemmParams& p, const int* s_prefix, const int* s_mm, int t,
                                          int& gcur, Tile& c, uint32_t lane) {
    if constexpr (KIND == kMasked) {
        return masked_tile(s_prefix, s_mm, p.groups, t, gcur, c);
    } else {
        if (!raster_tile(p, t, c)) return false;
        if constexpr (KIND == kContiguous && NEED_EXPERT) c.g = block_expert(p, c.m_blk, lane);
        return true;
    }
}

// ------------------------------------------------------- scale-word gather --

// Scale words of one 4-K-block group for a tile: lane r holds, for j = 0..3,
// the word of A row 32j + r and, per 128-column chunk, the word of B column
// 128*chunk + 32j + r. Stored as one 16-byte row per lane, this is the
// 32x128-bit matrix whose copy to TMEM puts row m at lane m % 32, column m / 32.
template <int BN, int KIND>
struct ScaleWords {
    static constexpr int CH = GemmConfig<BN>::SFB_CHUNKS;
    uint32_t a[4];
    uint32_t b[CH][4];

    __device__ __forceinline__ void load(const GemmParams& p, const Tile& c, int kg, uint32_t lane) {
        // A rows: clamp into the operand so every load is in bounds; rows past
        // the valid count only feed accumulator rows that are never stored.
        size_t row_base = 0;
        int row_lim = p.rows;
        if constexpr (KIND == kMasked) row_base = static_cast<size_t>(c.g) * p.rows;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = min(c.m_blk * BM + 32 * j + static_cast<int>(lane), row_lim - 1);
            a[j] = static_cast<uint32_t>(__ldg(p.sfa + (row_base + r) * p.kp + kg));
        }
        const int g = (KIND == kDense) ? 0 : max(c.g, 0);
        const int32_t* sfb = p.sfb + static_cast<size_t>(g) * p.nb_sf * p.kp;
#pragma unroll
        for (int ch = 0; ch < CH; ++ch) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int col = c.n_blk * BN + 128 * ch + 32 * j + static_cast<int>(lane);
                const int nb = min(col / 128, p.nb_sf - 1);
                b[ch][j] = static_cast<uint32_t>(__ldg(sfb + static_cast<size_t>(nb) * p.kp + kg));
            }
        }
    }

    __device__ __forceinline__ void store(uint8_t* sfa_slot, uint8_t* sfb_slot, uint32_t lane) const {
        reinterpret_cast<uint4*>(sfa_slot)[lane] = make_uint4(a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int ch = 0; ch < CH; ++ch)
            reinterpret_cast<uint4*>(sfb_slot + 512 * ch)[lane] = make_uint4(b[ch][0], b[ch][1], b[ch][2], b[ch][3]);
    }
};

// ------------------------------------------------------------------ kernel --

template <int BN, int KIND>
__global__ void __launch_bounds__(NUM_THREADS, 1) fp8_block_scaled_gemm_kernel(const __grid_constant__ GemmParams p) {
    using Cfg = GemmConfig<BN>;
    constexpr int STAGES = Cfg::STAGES;
    constexpr int NUM_ACC = Cfg::NUM_ACC;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* smem_a = smem;                                         // STAGES x 16 KB
    uint8_t* smem_b = smem_a + STAGES * Cfg::A_BYTES;               // STAGES x BN*128
    uint8_t* smem_epi = smem_b + STAGES * Cfg::B_BYTES;             // 4 warps x 2 x 2 KB (1024-aligned)
    uint8_t* smem_sfa = smem_epi + Cfg::EPI_BYTES;                  // STAGES x 512
    uint8_t* smem_sfb = smem_sfa + STAGES * Cfg::SFA_BYTES;         // STAGES x 512*chunks
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem_sfb + STAGES * Cfg::SFB_BYTES);
    uint64_t* full_bar = bars;                    // TMA bytes + scale words landed
    uint64_t* empty_bar = bars + STAGES;          // MMAs reading the stage finished
    uint64_t* tfull_bar = bars + 2 * STAGES;      // accumulator ready for the epilogue
    uint64_t* tempty_bar = tfull_bar + 2;         // accumulator drained by the epilogue
    uint64_t* drain_bar = tempty_bar + 2;         // all MMAs of this CTA finished
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain_bar + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    int* s_prefix = reinterpret_cast<int*>(s_tmem + 4);             // [groups + 1]
    int* s_mm = s_prefix + MAX_MASKED_GROUPS + 4;                   // [groups]

    const uint32_t warp = threadIdx.x / 32;
    const uint32_t lane = lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull_bar[i], 1);
            mbar_init(&tempty_bar[i], 4);
        }
        mbar_init(drain_bar, 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.tma_a);
        tma_prefetch_desc(&p.tma_b);
        tma_prefetch_desc(&p.tma_d);
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    if constexpr (KIND == kMasked) {
        // masked_m clamped to [0, max_m]; tile prefix over groups (warp 0 scans).
        for (int g = threadIdx.x; g < p.groups; g += NUM_THREADS) s_mm[g] = min(max(__ldg(p.meta + g), 0), p.rows);
        __syncthreads();
        if (warp == 0) {
            const int per = (p.groups + 31) / 32;
            const int g0 = static_cast<int>(lane) * per;
            int sum = 0;
            for (int i = 0; i < per; ++i) {
                const int g = g0 + i;
                if (g < p.groups) sum += ((s_mm[g] + BM - 1) / BM) * p.num_n_blocks;
            }
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= static_cast<uint32_t>(o)) incl += v;
            }
            int run = incl - sum;
            for (int i = 0; i < per; ++i) {
                const int g = g0 + i;
                if (g < p.groups) {
                    s_prefix[g] = run;
                    run += ((s_mm[g] + BM - 1) / BM) * p.num_n_blocks;
                }
            }
            if (lane == 31) s_prefix[p.groups] = incl;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;

    if (warp == 0) {
        // ------------------------------------------------------- producer --
        const int kg_count = (p.kb + 3) / 4;
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        int gcur = 0, gcur_ahead = 0;
        Tile cur, ahead;
        bool have = next_tile<KIND, true>(p, s_prefix, s_mm, blockIdx.x, gcur, cur, lane);
        // Scale words of the next group to store. Their loads are issued one
        // group (four stages) before they are needed, so the global-load
        // latency hides behind the TMA traffic of those stages.
        ScaleWords<BN, KIND> sw;
        int ahead_t = blockIdx.x, ahead_kg = 0;
        bool ahead_ok = have;
        if (have) {
            ahead = cur;
            gcur_ahead = gcur;
            sw.load(p, ahead, 0, lane);
        }
        bool aborted = false;
        for (int t = blockIdx.x; have; t += gridDim.x) {
            const int b_row = cur.n_blk * BN;
            const int g = max(cur.g, 0);
            for (int kb = 0; kb < p.kb; ++kb) {
                if (!wait_bounded(&empty_bar[stage], phase ^ 1u, p, s_abort)) { aborted = true; break; }
                const bool sf_stage = (kb & 3) == 0;
                if (lane == 0) {
                    constexpr uint32_t bytes = Cfg::A_BYTES + Cfg::B_BYTES;
                    if (sf_stage) mbar_expect_tx(&full_bar[stage], bytes);
                    else mbar_arrive_expect_tx(&full_bar[stage], bytes);
                    uint8_t* a_dst = smem_a + stage * Cfg::A_BYTES;
                    uint8_t* b_dst = smem_b + stage * Cfg::B_BYTES;
                    const int kx = kb * BK;
                    if constexpr (KIND == kMasked) {
                        tma_load_3d(a_dst, &p.tma_a, &full_bar[stage], kx, cur.m_blk * BM, cur.g);
                    } else {
                        tma_load_2d(a_dst, &p.tma_a, &full_bar[stage], kx, cur.m_blk * BM);
                    }
                    if constexpr (KIND == kDense) {
                        tma_load_2d(b_dst, &p.tma_b, &full_bar[stage], kx, b_row);
                    } else {
                        tma_load_3d(b_dst, &p.tma_b, &full_bar[stage], kx, b_row, g);
                    }
                }
                if (sf_stage) {
                    sw.store(smem_sfa + stage * Cfg::SFA_BYTES, smem_sfb + stage * Cfg::SFB_BYTES, lane);
                    fence_proxy_async_smem();
                    __syncwarp();
                    // test hook: CTA 0 withholds the arrive of its first stage
                    const bool withhold = p.test_mode == 1 && blockIdx.x == 0 && issued == 0;
                    if (lane == 0 && !withhold) mbar_arrive(&full_bar[stage]);
                    // start the loads of the following group
                    if (ahead_ok) {
                        if (++ahead_kg == kg_count) {
                            ahead_kg = 0;
                            ahead_t += gridDim.x;
                            ahead_ok = next_tile<KIND, true>(p, s_prefix, s_mm, ahead_t, gcur_ahead, ahead, lane);
                        }
                        if (ahead_ok) sw.load(p, ahead, ahead_kg, lane);
                    }
                }
                __syncwarp();
                ++issued;
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (aborted) break;
            have = next_tile<KIND, true>(p, s_prefix, s_mm, t + gridDim.x, gcur, cur, lane);
        }
        if (aborted) {
            // let the loads already issued land before shared memory goes away
            int s = stage;
            uint32_t ph = phase;
            for (int i = 0; i < STAGES && i < issued; ++i) {
                if (--s < 0) { s = STAGES - 1; ph ^= 1u; }
                wait_quiet(&full_bar[s], ph, p.wait_limit_ns / 16);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA --
        constexpr uint32_t IDESC = idesc_mxf8_e4m3_ue8m0(BN);
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        int gcur = 0;
        Tile c;
        bool aborted = false;
        for (int t = blockIdx.x; !aborted && next_tile<KIND, false>(p, s_prefix, s_mm, t, gcur, c, lane); t += gridDim.x) {
            if (!wait_bounded(&tempty_bar[acc], acc_phase ^ 1u, p, s_abort)) { aborted = true; break; }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + acc * Cfg::ACC_COLS;
            for (int kb = 0; kb < p.kb; ++kb) {
                if (!wait_bounded(&full_bar[stage], phase, p, s_abort)) { aborted = true; break; }
                tc_fence_after();
                if (lane == 0) {
                    if ((kb & 3) == 0) {
                        tc_cp_32x128b_warpx4(tmem_base + Cfg::SFA_COL,
                                             smem_desc_sf(smem_u32(smem_sfa + stage * Cfg::SFA_BYTES)));
#pragma unroll
                        for (int ch = 0; ch < Cfg::SFB_CHUNKS; ++ch)
                            tc_cp_32x128b_warpx4(tmem_base + Cfg::SFB_COL + 4 * ch,
                                                 smem_desc_sf(smem_u32(smem_sfb + stage * Cfg::SFB_BYTES + 512 * ch)));
                    }
                    const uint32_t sf_id = static_cast<uint32_t>(kb & 3);
                    const uint32_t idesc = idesc_with_sf_id(IDESC, sf_id);
                    const uint32_t sfa_t = (tmem_base + Cfg::SFA_COL) | (sf_id << 30);
                    const uint32_t sfb_t = (tmem_base + Cfg::SFB_COL) | (sf_id << 30);
                    const uint64_t adesc = smem_desc_sw128(smem_u32(smem_a + stage * Cfg::A_BYTES));
                    const uint64_t bdesc = smem_desc_sw128(smem_u32(smem_b + stage * Cfg::B_BYTES));
#pragma unroll
                    for (int k = 0; k < BK / MMA_K; ++k) {
                        // advance the start address by 32 bytes of K inside the swizzled row
                        const uint64_t koff = static_cast<uint64_t>((k * MMA_K) >> 4);
                        tc_mma_mxf8f6f4_block_scale(d_tmem, adesc + koff, bdesc + koff, idesc, sfa_t, sfb_t,
                                                    (kb > 0 || k > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty_bar[stage]);
                }
                __syncwarp();
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (aborted) break;
            if (lane == 0) tc_commit(&tfull_bar[acc]);
            __syncwarp();
            if (++acc == NUM_ACC) { acc = 0; acc_phase ^= 1u; }
        }
        // all MMAs of this CTA must finish before TMEM is released
        if (lane == 0) tc_commit(drain_bar);
        __syncwarp();
        wait_quiet(drain_bar, 0, p.wait_limit_ns);
    } else {
        // ------------------------------------------------------- epilogue --
        // Each warp owns 32 rows (its TMEM sub-partition). Per tile it reads
        // the accumulator in batches of up to 128 columns, hands TMEM back to
        // the MMA warp right after the last read, and then writes bf16:
        // 32x32 chunks staged in swizzled shared memory and stored with TMA
        // when all 32 rows may be written, predicated 16-byte stores otherwise.
        const int q = static_cast<int>(warp & 3);   // TMEM sub-partition of this warp
        uint8_t* stg = smem_epi + (warp - 2) * Cfg::EPI_WARP_BYTES;
        int acc = 0;
        uint32_t acc_phase = 0;
        int gcur = 0;
        int buf = 0;
        Tile c;
        for (int t = blockIdx.x; next_tile<KIND, true>(p, s_prefix, s_mm, t, gcur, c, lane); t += gridDim.x) {
            const int mloc = c.m_blk * BM + 32 * q + static_cast<int>(lane);
            bool valid;
            size_t out_row;
            if constexpr (KIND == kDense) {
                valid = mloc < p.rows;
                out_row = static_cast<size_t>(mloc);
            } else if constexpr (KIND == kMasked) {
                valid = mloc < s_mm[c.g];
                out_row = static_cast<size_t>(c.g) * p.rows + mloc;
            } else {
                const int id = (mloc < p.rows) ? __ldg(p.meta + mloc) : -1;
                const bool in_range = id >= 0 && id < p.groups;
                valid = in_range && id == c.g;
                if (in_range && id != c.g) atomicOr(p.status, DEVERR_MIXED_EXPERT_BLOCK);
                out_row = static_cast<size_t>(mloc);
            }
            // TMA stores clip at the tensor's edges, so for the dense form rows
            // past M are safe; the grouped forms need every row of the chunk valid.
            const bool use_tma = (KIND == kDense) ? true : (__all_sync(0xffffffffu, valid) != 0);
            const int row_coord = c.m_blk * BM + 32 * q;
            if (!wait_bounded(&tfull_bar[acc], acc_phase, p, s_abort)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + acc * Cfg::ACC_COLS;
            const int n0 = c.n_blk * BN;
            __nv_bfloat16* drow = p.d + out_row * static_cast<size_t>(p.n) + n0;
#pragma unroll
            for (int h = 0; h < BN; h += 128) {
                constexpr int kMaxBatch = 128;
                const int cols = (BN - h) < kMaxBatch ? (BN - h) : kMaxBatch;  // compile-time after unrolling
                uint32_t r[kMaxBatch];
#pragma unroll
                for (int j = 0; j < kMaxBatch / 32; ++j)
                    if (32 * j < cols) tmem_ld_32x32b_x32(taddr + h + 32 * j, r + 32 * j);
                tc_wait_ld();
                if (h + 128 >= BN) {
                    // last TMEM read of this accumulator: hand it back to the MMA warp
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty_bar[acc]);
                }
#pragma unroll
                for (int j = 0; j < kMaxBatch / 32; ++j) {
                    if (32 * j >= cols) continue;
                    const int col = n0 + h + 32 * j;
                    if (col >= p.n) continue;  // warp-uniform: N tail
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[32 * j + 2 * i]),
                                                                  __uint_as_float(r[32 * j + 2 * i + 1]));
                        w[i] = *reinterpret_cast<uint32_t*>(&b2);
                    }
                    if (use_tma) {
                        // the store issued two chunks ago has finished reading this buffer
                        if (lane == 0) bulk_wait_group_read<1>();
                        __syncwarp();
                        uint8_t* sb = stg + buf * 2048;
                        // 32 rows x 64 bytes with the 64-byte swizzle: granule g of
                        // row r sits at granule g ^ ((r >> 1) & 3)
                        const uint32_t sw = (lane >> 1) & 3u;
#pragma unroll
                        for (int g = 0; g < 4; ++g)
                            *reinterpret_cast<uint4*>(sb + lane * 64 + 16 * (g ^ sw)) =
                                make_uint4(w[4 * g], w[4 * g + 1], w[4 * g + 2], w[4 * g + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            if constexpr (KIND == kMasked) tma_store_3d(&p.tma_d, sb, col, row_coord, c.g);
                            else tma_store_2d(&p.tma_d, sb, col, row_coord);
                            bulk_commit_group();
                        }
                        buf ^= 1;
                    } else if (valid) {
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            if (col + 8 * v < p.n)
                                *reinterpret_cast<uint4*>(drow + h + 32 * j + 8 * v) =
                                    make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
                    }
                }
            }
            if (++acc == NUM_ACC) { acc = 0; acc_phase ^= 1u; }
        }
        // every bulk store must have completed before the CTA exits
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace dg
