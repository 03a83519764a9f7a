// Persistent, warp-specialised FP8 block-scaled GEMM for sm_100a.
//
// D = A . B^T with E4M3 operands, packed UE8M0 scales (one per 1x128 block of
// A, one per 128x128 block of B or one per 1x128 block of each row of B),
// fp32 accumulation in TMEM, bf16 output. One template serves the forms of the
// method ("DeepInside DeepGEMM" section 4 for the dense NT GEMM; "DeepGEMM CUDA
// Graph Compatibility for Masked Grouped GEMMs" for the masked form and for
// the groups given by psum_m; the contiguous form is the "continuous storage
// layout" of "DeepGEMM tested by Novita AI"), and also the BF16 masked GEMM.
//
// CTA = 7 warps, one CTA per SM, persistent over a grid fixed by the sizes:
//   warp 0      TMA producer: loads of the A and B tiles (128-byte swizzle)
//               into a STAGES-deep shared-memory ring.
//   warp 6      scale producer: per group of four K-blocks (one packed int32
//               per row/column) gathers the scale words into the 32x16-byte
//               layout that tcgen05.cp expects, into its own 4-deep ring, with
//               the loads of the next two groups in flight.
//   warp 1      MMA issuer: allocates TMEM, copies each group's scale words to
//               TMEM (and frees their slot as soon as the copy completes),
//               issues tcgen05.mma.kind::mxf8f6f4.block_scale (K=32) four
//               times per 128-K block, selecting the UE8M0 byte of the
//               current K-block with the scale-factor id, and commits stage
//               releases and accumulator hand-offs to mbarriers.
//   warps 2..5  epilogue: TMEM -> registers (tcgen05.ld, up to 128 columns
//               per batch; TMEM is handed back right after the last read),
//               fp32 -> bf16 with round-to-nearest-even, 32x32 chunks staged
//               in swizzled shared memory and written by TMA; chunks holding
//               rows that must not be written (past masked_m, padding of
//               m_indices, past a psum_m group's end) use predicated row
//               stores instead, so those rows are never touched.
// Every role runs its loop on the whole warp: waits are warp-wide votes and
// the TMA / tcgen05 instructions are issued by one lane chosen with
// elect.sync. (A loop run by one lane, or guarded by a lane test, leaves the
// tensor pipe idle for part of every K-block: each barrier probe then holds up
// the MMAs issued after it.)
// The accumulator is double-buffered in TMEM when two fit next to the scale
// columns, so the epilogue of tile i overlaps the MMAs of tile i+1.
//
// CG = 2 runs a cluster of two CTAs as one MMA unit (tcgen05 cta_group::2):
// a 256 x BN tile whose A rows are split 128/128 and whose B rows are split
// BN/2 / BN/2 between the two CTAs' shared memory. Only the even CTA (the
// leader) issues MMAs and tcgen05 copies (all with cta_group::2); both CTAs'
// TMA loads complete on the leader's stage barrier, the leader's scale warp
// gathers both CTAs' scale words and writes the peer's share into the peer's
// shared memory (so that hand-off stays inside the leader), and commits reach
// both CTAs' barriers. Each CTA's TMEM holds its 128 rows x BN of the
// accumulator, its own A scales and the full-width B scales. Per SM this
// halves the B bytes each 128-K block needs, which is what bounds a single
// CTA: the L2 feeds an SM about 77 bytes per clock, so a 128 x 224 tile
// (44 KB per K-block) waits on loads while a pair's 30 KB per SM does not.
// No load is multicast.
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
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda.h>

#include "ptx.cuh"

namespace dg {

// kPsum: groups given by psum_m, the inclusive prefix sums of their row counts
// (group g owns rows [psum_m[g-1], psum_m[g]) of an unpadded A).
enum GemmKind : int { kDense = 0, kContiguous = 1, kMasked = 2, kPsum = 3 };
// Operand type: E4M3 with packed UE8M0 block scales, or plain BF16 (no scales).
enum OperandType : int { kE4M3 = 0, kBF16 = 1 };

constexpr int BM = 128;                 // rows of A per CTA
constexpr int BK = 128;                 // bytes of K per pipeline stage (E4M3: 128 values = one scale block)
constexpr int NUM_THREADS = 224;
constexpr int SF_RING = 4;              // scale-word groups in flight
constexpr int MAX_MASKED_GROUPS = 1024;
constexpr int MAX_CACHED_BLOCKS = 1024;  // contiguous: 128-row blocks whose expert is kept in shared memory
constexpr int SMEM_LIMIT = 232448;      // 227 KB opt-in per CTA
constexpr uint64_t DEFAULT_WAIT_LIMIT_NS = 2000000000ull;  // 2 s

constexpr uint32_t DEVERR_TIMEOUT = 1u;
constexpr uint32_t DEVERR_MIXED_EXPERT_BLOCK = 2u;

constexpr int SPLIT_NONE = 0;
constexpr int SPLIT_SCRATCH = 1;
constexpr int SPLIT_CLUSTER = 2;
constexpr int MAX_CLUSTER_SPLITS = 8;   // portable cluster size

struct GemmParams {
    CUtensorMap tma_a;        // A: 2-D {K, rows} (dense, contiguous, psum_m) or 3-D {K, max_m, G} (masked)
    CUtensorMap tma_b;        // B: 2-D {K, N} (dense) or 3-D {K, N, G} (grouped); box BN/CG rows
    CUtensorMap tma_d;        // D (store): 2-D {N, rows} or 3-D {N, max_m, G}; bf16: 32x32 boxes, 64-byte
                              //   swizzle; fp32 (dense): 32 columns x 16 rows, 128-byte swizzle
    CUtensorMap tma_c;        // C of D = C + A.B^T (load), D's type and box; set when c is given
    const int32_t* sfa;       // packed scale rows of A
    const int32_t* sfb;       // packed scale rows of B (per 128 rows or per row, per group)
    __nv_bfloat16* d;         // output
    const int32_t* meta;      // m_indices (contiguous) / masked_m (masked) / psum_m (psum_m) / null
    uint32_t* status;         // device status word
    int rows;                 // M (dense), M_total (contiguous, psum_m), max_m (masked)
    int n, k, groups;
    int kb;                   // K / 128
    int kp;                   // ceil(kb / 4) packed words per scale row
    int nb_sf;                // scale rows per weight matrix: ceil(N / 128), or N when sfb_per_row
    int sfb_per_row;          // 1: one scale row per row of B (1x128 blocks); 0: per 128x128 block
    int num_m_blocks;         // ceil(rows / (128 * CG)) m-tiles
    int num_n_blocks;         // ceil(N / BN)
    int raster_group;         // m-tiles per raster band (dense / contiguous), a power of two
    int raster_shift;         // log2(raster_group)
    float inv_band_tiles;     // 1 / (raster_group * num_n_blocks), for the band index
    uint64_t wait_limit_ns;   // bound of every mbarrier wait
    int k_rotate;             // 1: each tile walks its K groups starting at group (tile mod groups)
    int test_mode;            // 1: CTA 0 withholds its first scale-group arrive (exercises the timeout path)
    int sf_vec4;              // 1: scale rows are read 16 bytes (4 K groups) at a time (B scaled per row,
                              //    kp % 4 == 0, 16-byte bases, K groups in order)
    // split-K (dense form, single CTAs): each output tile is computed by `splits`
    // work units over disjoint ranges of K groups, whose fp32 partials are
    // added in split order
    int splits;               // 1 = no split; range i covers K groups [i*G/splits, (i+1)*G/splits)
    int split_mode;           // SPLIT_CLUSTER: the units of a tile form one cluster and add their
                              //   partials through distributed shared memory (no global scratch);
                              // SPLIT_SCRATCH: units park partials in `ws` and the last one to
                              //   finish adds them
    float* ws;                // SPLIT_SCRATCH partials: [tile][split][4 row quarters][BN/4][32 lanes][4]
    uint32_t* counters;       // SPLIT_SCRATCH: finished units per output tile; zero between calls
    // dense form: D = C + A.B^T. C (optional, [rows, n] in D's type) is added to
    // the fp32 accumulation before the final conversion; D is bf16 (d, TMA
    // stores) or fp32 (d32, direct stores)
    const void* c;
    float* d32;
    int out_f32;
};

// SCHED_INTS: 32-bit words of shared memory for the tile scheduler (masked:
// clamped masked_m and tile prefix sums; psum_m: the groups' first rows and
// tile prefix sums; contiguous: expert of every 128-row block; dense: none).
template <int KIND>
__host__ __device__ constexpr int sched_ints() {
    return (KIND == kMasked || KIND == kPsum) ? 2 * MAX_MASKED_GROUPS + 8
                                             : (KIND == kContiguous ? MAX_CACHED_BLOCKS + 8 : 16);
}

// A_ROWS: rows of A per stage. 128 normally; 64 for the dense form when M <= 64
// (a 64-row TMA box; the MMA still reads 128 rows, and its other 64 rows read
// the next 8 KB of shared memory, whose accumulator rows are never stored).
// The smaller stage keeps more weight bytes in flight per SM.
template <int BN, int CG, int SCHED_INTS, int DT = kE4M3, int A_ROWS = BM>
struct GemmConfig {
    static_assert(A_ROWS == BM || A_ROWS == 64, "A stages of 128 or 64 rows");
    static_assert(BN % 16 == 0 && BN >= 32 && BN <= 256, "N tile must be a multiple of 16 in [32, 256]");
    static_assert(BN % 32 == 0 || CG == 2, "tiles with a 16-column tail chunk are built for CTA pairs");
    static_assert(CG == 1 || CG == 2, "one CTA or a CTA pair");
    static constexpr int B_ROWS = BN / CG;                      // rows of B in this CTA's shared memory
    static constexpr int A_BYTES = A_ROWS * BK;
    static constexpr int B_BYTES = B_ROWS * BK;
    static constexpr int SFB_CHUNKS = (BN + 127) / 128;         // 128-column chunks of B scales (full width)
    static constexpr int SFA_BYTES = 512;                       // 32 rows x 16 bytes
    static constexpr int SFB_BYTES = 512 * SFB_CHUNKS;
    static constexpr int SF_SLOT_BYTES = DT == kE4M3 ? SFA_BYTES + SFB_BYTES : 0;  // one group of scale words
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr uint32_t TX_BYTES = CG * (A_BYTES + B_BYTES);  // TMA bytes per stage, both CTAs
    static constexpr int EPI_WARP_BYTES = 2 * 2048;             // two 32x32 bf16 staging buffers per warp
    static constexpr int EPI_BYTES = 4 * EPI_WARP_BYTES;
    static constexpr int SCHED_BYTES = SCHED_INTS * 4;
    static constexpr int FIXED_BYTES =
        1024 /*align slack*/ + EPI_BYTES + SF_RING * SF_SLOT_BYTES + 512 /*barriers*/ + SCHED_BYTES;
    static constexpr int STAGES_FIT = (SMEM_LIMIT - FIXED_BYTES) / STAGE_BYTES;
    static constexpr int MAX_STAGES = A_ROWS < BM ? 16 : 8;
    static constexpr int STAGES = STAGES_FIT > MAX_STAGES ? MAX_STAGES : STAGES_FIT;
    static_assert(STAGES >= 2, "pipeline too shallow");
    static constexpr int SMEM_BYTES = FIXED_BYTES + STAGES * STAGE_BYTES;

    // TMEM columns: accumulator slot(s) of BN columns and two sets of scale
    // columns (4 of A scales and 4 per 128-column chunk of B scales), used by
    // alternate groups so that the copy of the next group's scales never
    // overwrites words that MMAs still in the pipe are reading. Widths that are
    // multiples of 32 put the slots side by side and the scale sets after them;
    // a width with a 16-column tail (BN = 240) keeps each slot on a 256-column
    // boundary and puts one scale set in the 16 columns after each slot.
    static constexpr int ACC_COLS = BN;
    static constexpr int SF_COLS = DT == kE4M3 ? 4 + 4 * SFB_CHUNKS : 0;
    static constexpr bool TAIL16 = BN % 32 != 0;
    static constexpr int ACC_STRIDE = TAIL16 ? 256 : BN;   // columns between accumulator slots
    static constexpr int NUM_ACC =
        TAIL16 ? ((256 - BN >= SF_COLS) ? 2 : 1) : ((2 * ACC_COLS + 2 * SF_COLS <= 512) ? 2 : 1);
    static constexpr int SF_SET0 = TAIL16 ? BN : NUM_ACC * ACC_COLS;
    static constexpr int SF_SET1 = TAIL16 ? 256 + BN : SF_SET0 + SF_COLS;
    static_assert(SF_SET1 + SF_COLS <= 512, "TMEM overflow");
    static_assert(!TAIL16 || NUM_ACC == 2, "a 16-column-tail tile is double-buffered");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t IDESC = DT == kE4M3 ? idesc_mxf8_e4m3_ue8m0(BM * CG, BN) : idesc_bf16_f32(BM * CG, BN);
    // K values per 128-byte row of a stage and per MMA instruction
    static constexpr int K_PER_STAGE = DT == kE4M3 ? 128 : 64;
};

struct Tile {
    int m_blk, n_blk, g;      // g: group (masked, psum_m) or expert (contiguous), 0 for dense
    int kg0, kg1;             // K groups [kg0, kg1) of this work unit
    int base, split;          // output tile index and split index (split-K; else base = t, split = 0)
    int e_own[2];             // contiguous: expert of each CTA's 128-row block (-1: padding only)
    int row0;                 // psum_m form: first row of A (and D) of the tile
};

// ----------------------------------------------------------------- waits ----

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of `bar` with the given parity, as a whole warp: every
// lane probes and the outcome is a vote, so all 32 lanes leave together with
// the same answer (a lane that left a loop early would leave the others
// waiting at the next elect.sync, __syncwarp or .sync.aligned instruction).
// Gives up when another role of this CTA has given up, or after
// p.wait_limit_ns; a timeout is recorded in the device status word.
// CLUSTER_ACQ: the probe acquires at cluster scope (the phase carries writes
// or arrives of other CTAs of the cluster).
template <bool CLUSTER_ACQ = false>
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, const GemmParams& p, volatile int* s_abort) {
    auto probe = [&]() { return CLUSTER_ACQ ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
    if (__all_sync(0xffffffffu, probe())) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (__all_sync(0xffffffffu, probe())) return true;
        const bool late = global_ns() - t0 > p.wait_limit_ns;
        if (__any_sync(0xffffffffu, late || *s_abort != 0)) {
            if (__any_sync(0xffffffffu, late) && lane_id() == 0) {
                atomicOr(p.status, DEVERR_TIMEOUT);
                *s_abort = 1;
            }
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

__device__ __forceinline__ void sleep_ns(uint64_t ns) {
    const uint64_t t0 = global_ns();
    while (global_ns() - t0 < ns) {
    }
}

// ------------------------------------------------------------- scheduling --

// Dense / contiguous: banded raster. Within a band of `raster_group` m-tiles
// the m-tile varies fastest, so CTAs running at the same time share the B tile
// and a bounded slab of A.
// The arithmetic is kept free of integer divisions where it can be (each
// costs ~0.1 us of a lone warp's time, paid between two tiles): no split
// needs none, the band index comes from a float reciprocal corrected to the
// exact quotient (below 2^20 tiles, where one correction step suffices), and
// full bands (a power-of-two number of m-tiles) use a shift.
__device__ __forceinline__ bool raster_tile(const GemmParams& p, int t_unit, Tile& c) {
    const int kgc = (p.kb + 3) / 4;  // K groups of four 128-K blocks
    int t = t_unit;                  // output tile; its splits are consecutive work units
    int split = 0;
    c.kg0 = 0;
    c.kg1 = kgc;
    if (p.splits > 1) {
        t = t_unit / p.splits;
        split = t_unit - t * p.splits;
        c.kg0 = split * kgc / p.splits;
        c.kg1 = (split + 1) * kgc / p.splits;
    }
    const int total = p.num_m_blocks * p.num_n_blocks;
    if (t >= total) return false;
    c.base = t;
    c.split = split;
    const int band_tiles = p.raster_group * p.num_n_blocks;
    int band;
    if (total < (1 << 20)) {
        band = __float2int_rz(__int2float_rn(t) * p.inv_band_tiles);
        if ((band + 1) * band_tiles <= t) ++band;
        if (band * band_tiles > t) --band;
    } else {
        band = t / band_tiles;
    }
    const int local = t - band * band_tiles;
    const int m0 = band * p.raster_group;
    const int gm = min(p.raster_group, p.num_m_blocks - m0);
    if (gm == p.raster_group) {
        c.n_blk = local >> p.raster_shift;
        c.m_blk = m0 + (local & (gm - 1));
    } else {
        c.n_blk = local / gm;
        c.m_blk = m0 + (local - c.n_blk * gm);
    }
    c.g = 0;
    return true;
}

// Rows of group g. Masked: s_mm[g] is the clamped masked_m. psum_m form: s_mm
// holds the groups' first rows (g = 0..groups), so group g has s_mm[g+1] - s_mm[g].
template <int KIND>
__device__ __forceinline__ int group_rows(const int* s_mm, int g) {
    if constexpr (KIND == kPsum) return s_mm[g + 1] - s_mm[g];
    else return s_mm[g];
}

// Masked and psum_m forms: tiles of group g are numbered from s_prefix[g];
// within a group the m-block varies fastest. `gcur` is the caller's monotone
// cursor.
template <int KIND>
__device__ __forceinline__ bool masked_tile(const int* s_prefix, const int* s_mm, int groups, int t, int& gcur,
                                            Tile& c) {
    if (t >= s_prefix[groups]) return false;
    while (s_prefix[gcur + 1] <= t) ++gcur;
    const int local = t - s_prefix[gcur];
    const int mb = (group_rows<KIND>(s_mm, gcur) + BM - 1) / BM;
    c.g = gcur;
    c.n_blk = local / mb;
    c.m_blk = local - c.n_blk * mb;
    c.base = t;
    c.split = 0;
    c.row0 = (KIND == kPsum ? s_mm[gcur] : 0) + c.m_blk * BM;
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

// block_expert from the shared-memory table built in the kernel's prologue
// when the blocks fit in it (warp-uniform either way).
__device__ __forceinline__ int cached_block_expert(const GemmParams& p, const int* s_bexp, int blk, uint32_t lane) {
    const int nblk = (p.rows + BM - 1) / BM;
    if (nblk <= MAX_CACHED_BLOCKS) return blk < nblk ? s_bexp[blk] : -1;
    return block_expert(p, blk, lane);
}

// Next work unit at or after t (stepping by `units`); false when none is left.
// Contiguous form on CTA pairs: a pair tile covers two 128-row blocks, which
// may belong to two experts (segments are 128-row aligned). Tiles are visited
// in two passes over (pair, n-block): pass 0 computes the pair with the first
// block's expert (the second block's if the first is padding only); pass 1
// exists only when the second block has another expert, and computes the pair
// with that one. Rows of the other expert are never written in a pass. Tiles
// of padding only are skipped. Every role of the CTA takes the same steps.
template <int KIND, bool NEED_EXPERT, int CG>
__device__ __forceinline__ bool next_tile(const GemmParams& p, const int* s_prefix, const int* s_mm, int& t,
                                          int units, int& gcur, Tile& c, uint32_t lane) {
    if constexpr (KIND == kMasked || KIND == kPsum) {
        c.kg0 = 0;
        c.kg1 = (p.kb + 3) / 4;
        return masked_tile<KIND>(s_prefix, s_mm, p.groups, t, gcur, c);
    } else if constexpr (KIND == kContiguous && CG == 2) {
        const int per_pass = p.num_m_blocks * p.num_n_blocks;
        for (; t < 2 * per_pass; t += units) {
            const int pass = t >= per_pass ? 1 : 0;
            raster_tile(p, t - pass * per_pass, c);
            const int e0 = cached_block_expert(p, s_prefix, 2 * c.m_blk, lane);
            const int e1 = cached_block_expert(p, s_prefix, 2 * c.m_blk + 1, lane);
            c.e_own[0] = e0;
            c.e_own[1] = e1;
            if (pass == 0) {
                c.g = e0 >= 0 ? e0 : e1;
                if (c.g >= 0) return true;
            } else if (e0 >= 0 && e1 >= 0 && e1 != e0) {
                c.g = e1;
                return true;
            }
        }
        return false;
    } else {
        if (!raster_tile(p, t, c)) return false;
        if constexpr (KIND == kContiguous && NEED_EXPERT) {
            c.g = cached_block_expert(p, s_prefix, c.m_blk, lane);
            c.e_own[0] = c.g;
        }
        return true;
    }
}

// Group of four K-blocks visited at step gi of tile t. Rotating the start by
// the tile index makes CTAs that share an A or B tile (and run in lockstep)
// touch its K-blocks at different times, so only one of them waits for DRAM
// per block and the others are served from L2. Whole groups keep the packed
// scale words aligned; only the order of the fp32 accumulation changes.
__device__ __forceinline__ int rot_group(const GemmParams& p, int t, int gi, int kg_count) {
    return p.k_rotate ? (gi + t) % kg_count : gi;
}

// ------------------------------------------------------- scale-word gather --

// Scale words of one 4-K-block group of a tile: lane r holds, for j = 0..3,
// the word of A row row0 + 32j + r and, per 128-column chunk, the word of B
// column n0 + 128*chunk + 32j + r (from the scale row of its 128x128 block, or
// its own scale row when B is scaled per row). Stored as one 16-byte row per lane, this is
// the 32x128-bit matrix whose copy to TMEM puts row m at lane m % 32, column
// m / 32. For a CTA pair (CG = 2) the words of the second CTA's 128 rows are
// gathered too (`ap`), by the leader, which stores them into the peer's slot.
template <int BN, int KIND, int CG>
struct ScaleWords {
    static constexpr int CH = (BN + 127) / 128;
    uint32_t a[4];
    uint32_t ap[CG == 2 ? 4 : 1];
    uint32_t b[CH][4];

    __device__ __forceinline__ void load(const GemmParams& p, int row0, int n0, int g, int kg, uint32_t lane) {
        // A rows: clamp into the operand so every load is in bounds; rows past
        // the valid count only feed accumulator rows that are never stored.
        size_t row_base = 0;
        if constexpr (KIND == kMasked) row_base = static_cast<size_t>(g) * p.rows;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = min(row0 + 32 * j + static_cast<int>(lane), p.rows - 1);
            a[j] = static_cast<uint32_t>(__ldg(p.sfa + (row_base + r) * p.kp + kg));
            if constexpr (CG == 2) {
                const int rp = min(row0 + BM + 32 * j + static_cast<int>(lane), p.rows - 1);
                ap[j] = static_cast<uint32_t>(__ldg(p.sfa + (row_base + rp) * p.kp + kg));
            }
        }
        load_b(p, n0, g, kg, lane);
    }

    // B's words of group kg only
    __device__ __forceinline__ void load_b(const GemmParams& p, int n0, int g, int kg, uint32_t lane) {
        const int32_t* sfb = p.sfb + static_cast<size_t>(KIND == kDense ? 0 : max(g, 0)) * p.nb_sf * p.kp;
#pragma unroll
        for (int ch = 0; ch < CH; ++ch) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int col = n0 + 128 * ch + 32 * j + static_cast<int>(lane);
                const int nb = min(p.sfb_per_row ? col : col / 128, p.nb_sf - 1);
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

    // The peer CTA's copy of the slot (pairs): its A rows and the same B words,
    // written through the cluster window at the same shared-memory offsets.
    __device__ __forceinline__ void store_peer(uint32_t sfa_slot_peer, uint32_t sfb_slot_peer, uint32_t lane) const {
        if constexpr (CG == 2) {
            st_cluster_v4(sfa_slot_peer + 16u * lane, ap[0], ap[1], ap[2], ap[3]);
#pragma unroll
            for (int ch = 0; ch < CH; ++ch)
                st_cluster_v4(sfb_slot_peer + 512u * ch + 16u * lane, b[ch][0], b[ch][1], b[ch][2], b[ch][3]);
        }
    }
};

// Scale words of four consecutive K groups (one 16-byte load per scale row),
// for packed rows whose length is a multiple of four words on 16-byte
// aligned bases. Same rows and columns as ScaleWords; `base` is the first of
// the four groups (a multiple of 4). One such load serves four groups, so the
// scattered row reads are a quarter of the one-word loads: this pays for A's
// rows, and for B's when B is scaled per row (every column reads its own
// scale row). With 128x128 B blocks the B words, one broadcast word per 128
// columns, are read per group (`words` calls ScaleWords::load_b).
template <int BN, int KIND, int CG>
struct ScaleQuads {
    static constexpr int CH = (BN + 127) / 128;
    uint4 a[4];
    uint4 ap[CG == 2 ? 4 : 1];
    uint4 b[CH][4];
    int lo, hi;  // the groups [lo, hi) of the tile that this quad serves
    int n0, g;   // the tile's first column and group

    __device__ __forceinline__ static const uint4* at(const int32_t* row_start, int base) {
        return reinterpret_cast<const uint4*>(row_start + base);
    }

    __device__ __forceinline__ void load(const GemmParams& p, int row0, int n0, int g, int base, uint32_t lane) {
        size_t row_base = 0;
        if constexpr (KIND == kMasked) row_base = static_cast<size_t>(g) * p.rows;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = min(row0 + 32 * j + static_cast<int>(lane), p.rows - 1);
            a[j] = __ldg(at(p.sfa + (row_base + r) * p.kp, base));
            if constexpr (CG == 2) {
                const int rp = min(row0 + BM + 32 * j + static_cast<int>(lane), p.rows - 1);
                ap[j] = __ldg(at(p.sfa + (row_base + rp) * p.kp, base));
            }
        }
        this->n0 = n0;
        this->g = g;
        if (!p.sfb_per_row) return;  // B words are read per group
        const int32_t* sfb = p.sfb + static_cast<size_t>(KIND == kDense ? 0 : max(g, 0)) * p.nb_sf * p.kp;
#pragma unroll
        for (int ch = 0; ch < CH; ++ch) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int col = n0 + 128 * ch + 32 * j + static_cast<int>(lane);
                const int nb = min(p.sfb_per_row ? col : col / 128, p.nb_sf - 1);
                b[ch][j] = __ldg(at(sfb + static_cast<size_t>(nb) * p.kp, base));
            }
        }
    }

    __device__ __forceinline__ static uint32_t pick(const uint4& v, int i) {
        return static_cast<uint32_t>(i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w)));
    }

    // the words of group base + i (kg)
    __device__ __forceinline__ void words(const GemmParams& p, ScaleWords<BN, KIND, CG>& w, int i, int kg,
                                          uint32_t lane) const {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            w.a[j] = pick(a[j], i);
            if constexpr (CG == 2) w.ap[j] = pick(ap[j], i);
        }
        if (!p.sfb_per_row) {
            w.load_b(p, n0, g, kg, lane);
            return;
        }
#pragma unroll
        for (int ch = 0; ch < CH; ++ch)
#pragma unroll
            for (int j = 0; j < 4; ++j) w.b[ch][j] = pick(b[ch][j], i);
    }
};

// -------------------------------------------------- cluster split-K epilogue --
//
// SPLIT_CLUSTER: the `splits` = S units of an output tile are the S CTAs of one
// cluster; CTA r holds the fp32 partial of K range r of the whole 128 x BN
// tile in TMEM. The tile's columns are dealt out in 8-column pieces: of the
// NP = BN/8 pieces, CTA r owns [r*NP/S, (r+1)*NP/S). Each CTA sends every piece
// it does not own to the owner with st.async into the owner's operand ring
// (idle once the owner's own MMAs have completed), counted in bytes on the
// owner's barrier of the receiving epilogue warp. The owner adds the S
// partials of its pieces in split order, its own read back from TMEM, and
// writes them. Nothing outside the cluster's shared memory is used, so
// concurrent calls share no state.
//
// Layout of the received pieces in the owner's ring (16-byte units):
// [sender rank][piece j of the owner][half: columns 0-3 / 4-7][tile row].
__device__ __forceinline__ uint32_t cluster_piece_offset(int sender, int pmax, int j, int half, int row) {
    return static_cast<uint32_t>((((sender * pmax + j) * 2 + half) * BM + row) * 16);
}

// Shared-memory bytes of the received pieces of one tile: S slots of at most
// ceil(NP / S) pieces of 128 rows x 32 bytes.
__host__ __device__ constexpr int cluster_split_bytes(int bn, int splits) {
    return splits * ((bn / 8 + splits - 1) / splits) * BM * 32;
}

// Rows of the tile that the epilogue warp covering tile rows 32q..32q+31 must
// reduce: false when all of them lie past M (nothing to send or receive).
__device__ __forceinline__ bool cluster_warp_live(const GemmParams& p, int m_blk, int q) {
    return m_blk * BM + 32 * q < p.rows;
}

// Bytes the owner's warp q receives: S - 1 senders x its pieces x 32 rows x 32 bytes.
__device__ __forceinline__ uint32_t cluster_expected_bytes(const GemmParams& p, int rank, int np, int m_blk, int q) {
    const int S = p.splits;
    const int mine = (rank + 1) * np / S - rank * np / S;
    return cluster_warp_live(p, m_blk, q) ? static_cast<uint32_t>((S - 1) * mine * 32 * 32) : 0u;
}

// Eight reduced columns of one row of D at element offset `at`: + C and an
// fp32 or bf16 (round to nearest even) store (EPI 1), or a bf16 store (EPI 0).
template <int EPI>
__device__ __forceinline__ void cluster_store8(const GemmParams& p, float* acc, size_t at) {
    if constexpr (EPI == 1) {
        if (p.c != nullptr) {
            if (p.out_f32) {
                const float4 x0 = *reinterpret_cast<const float4*>(static_cast<const float*>(p.c) + at);
                const float4 x1 = *reinterpret_cast<const float4*>(static_cast<const float*>(p.c) + at + 4);
                acc[0] += x0.x; acc[1] += x0.y; acc[2] += x0.z; acc[3] += x0.w;
                acc[4] += x1.x; acc[5] += x1.y; acc[6] += x1.z; acc[7] += x1.w;
            } else {
                const uint4 x = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.c) + at);
                const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int h2 = 0; h2 < 4; ++h2) {
                    const float2 c2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[h2]));
                    acc[2 * h2] += c2.x;
                    acc[2 * h2 + 1] += c2.y;
                }
            }
        }
        if (p.out_f32) {
            *reinterpret_cast<float4*>(p.d32 + at) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            *reinterpret_cast<float4*>(p.d32 + at + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
            return;
        }
    }
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&b2);
    }
    *reinterpret_cast<uint4*>(p.d + at) = make_uint4(w[0], w[1], w[2], w[3]);
}

// The reduction and store of one warp's 32 rows (dense form, single CTAs).
// Returns false when a wait gave up.
template <int BN, int EPI>
__device__ __forceinline__ bool cluster_split_epilogue(const GemmParams& p, const Tile& c, int q, uint32_t warp,
                                                       uint32_t lane, uint32_t taddr, uint8_t* ring,
                                                       uint64_t* red_free, uint64_t* red_full,
                                                       volatile int* s_abort) {
    constexpr int NP = BN / 8;
    const int S = p.splits;
    const int rank = static_cast<int>(cluster_ctarank());
    const int pmax = (NP + S - 1) / S;
    const int row = 32 * q + static_cast<int>(lane);      // tile row of this thread
    const int m = c.m_blk * BM + row;                      // row of D
    const bool live = cluster_warp_live(p, c.m_blk, q);    // warp-uniform
    // 1. this CTA's MMAs have completed (the caller saw the accumulator
    //    barrier), so its ring may take the peers' pieces: tell every peer
    if (warp == 2) {
        __syncwarp();
        if (static_cast<int>(lane) < S && static_cast<int>(lane) != rank)
            mbar_arrive_release_cluster(mapa_shared(smem_u32(red_free), lane));
    }
    // 2. every peer's ring is free
    if (!wait_warp<true>(red_free, 0, p, s_abort)) return false;
    // 3. send the pieces other CTAs own
    if (live) {
        const uint32_t ring_s = smem_u32(ring);
        const uint32_t bar_s = smem_u32(&red_full[q]);
#pragma unroll
        for (int h = 0; h < BN; h += 32) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(taddr + h, r);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int pc = h / 8 + i;
                const int o = ((pc + 1) * S - 1) / NP;   // owner of piece pc
                if (o == rank) continue;
                const int j = pc - o * NP / S;
                const uint32_t dst = mapa_shared(ring_s, static_cast<uint32_t>(o));
                const uint32_t bar = mapa_shared(bar_s, static_cast<uint32_t>(o));
                st_async_v4(dst + cluster_piece_offset(rank, pmax, j, 0, row), bar, r[8 * i], r[8 * i + 1],
                            r[8 * i + 2], r[8 * i + 3]);
                st_async_v4(dst + cluster_piece_offset(rank, pmax, j, 1, row), bar, r[8 * i + 4], r[8 * i + 5],
                            r[8 * i + 6], r[8 * i + 7]);
            }
        }
    }
    // 4. every peer's pieces for these rows have landed: add the S partials of
    //    each owned piece in split order and store
    if (!wait_warp<true>(&red_full[q], 0, p, s_abort)) return false;
    if (live) {
        const int mine0 = rank * NP / S;
        const int mine1 = (rank + 1) * NP / S;
        for (int pc = mine0; pc < mine1; ++pc) {
            const int j = pc - mine0;
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
            for (int s = 0; s < S; ++s) {
                float v[8];
                if (s == rank) {
                    uint32_t t[8];
                    tmem_ld_32x32b_x8(taddr + 8 * pc, t);
                    tc_wait_ld();
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(t[i]);
                } else {
                    const float4 lo = *reinterpret_cast<const float4*>(ring + cluster_piece_offset(s, pmax, j, 0, row));
                    const float4 hi = *reinterpret_cast<const float4*>(ring + cluster_piece_offset(s, pmax, j, 1, row));
                    v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
                    v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] += v[i];
            }
            const int col = c.n_blk * BN + 8 * pc;
            // N % 8 == 0: a piece is wholly inside or outside D
            if (col < p.n && m < p.rows) cluster_store8<EPI>(p, acc, static_cast<size_t>(m) * p.n + col);
            __syncwarp();
        }
    }
    return true;
}

// ------------------------------------------------------------------ kernel --

// LAYOUT bit 0: A is stored MN-major ([K, M], M contiguous); bit 1: B is
// stored MN-major ([K, N]). MN-major tiles are loaded as 128-byte swizzle
// atoms of M or N by K rows and described to the MMA as such.
// EPI 1: the epilogue of D = C + A.B^T (optional C, bf16 or fp32 D; dense form);
// EPI 0: plain bf16 D.
// AR: rows of A per stage (64: dense, M <= 64, NT, plain epilogue; see GemmConfig).
template <int BN, int KIND, int CG, int DT, int LAYOUT = 0, int EPI = 0, int AR = BM>
__global__ void __launch_bounds__(NUM_THREADS, 1) fp8_block_scaled_gemm_kernel(const __grid_constant__ GemmParams p) {
    static_assert(CG == 1 || (KIND != kMasked && KIND != kPsum), "CTA pairs are built for the dense and contiguous forms");
    static_assert(DT == kE4M3 || (KIND == kMasked && CG == 1), "BF16 operands are built for the masked form");
    static_assert(LAYOUT == 0 || (KIND == kDense && DT == kE4M3), "layouts: dense form");
    static_assert(!(LAYOUT & 2) || (BN / CG) % 128 == 0, "an MN-major B tile is whole 128-byte atoms per CTA");
    static_assert(EPI == 0 || (KIND == kDense && DT == kE4M3 && LAYOUT == 0), "C / fp32 epilogue: dense NT form");
    constexpr bool kMnA = (LAYOUT & 1) != 0;
    constexpr bool kMnB = (LAYOUT & 2) != 0;
    static_assert(AR == BM || (KIND == kDense && CG == 1 && DT == kE4M3 && LAYOUT == 0 && EPI == 0),
                  "64-row A stages: dense NT form, single CTAs, plain epilogue");
    using Cfg = GemmConfig<BN, CG, sched_ints<KIND>(), DT, AR>;
    // instruction descriptor with the operands' major modes
    constexpr uint32_t kIdesc = Cfg::IDESC | (kMnA ? (1u << 15) : 0u) | (kMnB ? (1u << 16) : 0u);
    // MN-major descriptor strides: one atom is 128 K-rows x 128 bytes of M or
    // N (one TMA box); groups of 8 K-rows are 1024 bytes apart (stride byte
    // offset), and consecutive atoms along M or N 16 KB apart (leading byte
    // offset), so one MMA reads a whole 256-column MN-major B tile (two atoms).
    constexpr uint32_t kMnAtomBytes = BK * 128;
    constexpr uint32_t kMnLbo = kMnAtomBytes;
    constexpr uint32_t kMnSbo = 8 * 128;
    constexpr int STAGES = Cfg::STAGES;
    constexpr int NUM_ACC = Cfg::NUM_ACC;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* smem_a = smem;                                         // STAGES x 16 KB (8 KB for 64-row A)
    uint8_t* smem_b = smem_a + STAGES * Cfg::A_BYTES;               // STAGES x B_ROWS*128
    uint8_t* smem_epi = smem_b + STAGES * Cfg::B_BYTES;             // 4 warps x 2 x 2 KB (1024-aligned)
    uint8_t* smem_sf = smem_epi + Cfg::EPI_BYTES;                   // SF_RING x (A scales, B scales)
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem_sf + SF_RING * Cfg::SF_SLOT_BYTES);
    uint64_t* full_bar = bars;                    // A/B bytes landed (the leader's counts both CTAs)
    uint64_t* empty_bar = bars + STAGES;          // MMAs reading the stage finished
    uint64_t* sf_full_bar = bars + 2 * STAGES;    // scale words of a group stored (every CTA of the unit)
    uint64_t* sf_empty_bar = sf_full_bar + SF_RING;  // scale words copied into TMEM
    uint64_t* tfull_bar = sf_empty_bar + SF_RING;    // accumulator ready for the epilogue
    uint64_t* tempty_bar = tfull_bar + 2;            // accumulator drained by the epilogue(s)
    uint64_t* drain_bar = tempty_bar + 2;            // all MMAs issued for this CTA finished
    uint64_t* epi_bar = drain_bar + 1;               // split-K: the four epilogue warps meet
    uint64_t* red_free = epi_bar + 1;                // cluster split-K: every peer's ring is free
    uint64_t* red_full = red_free + 1;               // cluster split-K: peers' pieces landed, per epilogue warp
    uint64_t* cbar = red_full + 4;                   // D = C + A.B^T: a C piece landed, per epilogue warp
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(cbar + 4);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    volatile int* s_last = reinterpret_cast<volatile int*>(s_tmem + 2);  // split-K: this unit reduces
    int* s_prefix = reinterpret_cast<int*>(s_tmem + 4);             // [groups + 1] (masked, psum_m)
    int* s_mm = s_prefix + MAX_MASKED_GROUPS + 4;                   // [groups] (masked), [groups + 1] (psum_m)
    int* s_bexp = s_prefix;                                          // [128-row blocks] (contiguous)

    const uint32_t warp = threadIdx.x / 32;
    const uint32_t lane = lane_id();
    const uint32_t rank = (CG == 1) ? 0u : cluster_ctarank();    // position in the CTA pair
    const bool leader = rank == 0;
    const int unit = static_cast<int>(blockIdx.x) / CG;             // tile walker index (pair index)
    const int units = static_cast<int>(gridDim.x) / CG;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);           // the (leader's) arrive.expect_tx
            mbar_init(&empty_bar[s], 1);
        }
        for (int j = 0; j < SF_RING; ++j) {
            mbar_init(&sf_full_bar[j], 1);        // the scale producer (the leader's, for a pair)
            mbar_init(&sf_empty_bar[j], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull_bar[i], 1);
            mbar_init(&tempty_bar[i], 4 * CG);    // every epilogue warp of the unit
        }
        mbar_init(drain_bar, 1);
        mbar_init(epi_bar, 4);
        if constexpr (EPI == 1)
            for (int q = 0; q < 4; ++q) mbar_init(&cbar[q], 1);
        if constexpr (KIND == kDense && CG == 1) {
            if (p.split_mode == SPLIT_CLUSTER) {
                // one arrive from each peer; per epilogue warp, one arrive (made
                // here) plus the bytes the peers' pieces will bring
                mbar_init(red_free, static_cast<uint32_t>(p.splits - 1));
                Tile t0;
                raster_tile(p, static_cast<int>(blockIdx.x), t0);
                const int rk = static_cast<int>(cluster_ctarank());
                for (int q = 0; q < 4; ++q) {
                    mbar_init(&red_full[q], 1);
                    mbar_arrive_expect_tx(&red_full[q], cluster_expected_bytes(p, rk, BN / 8, t0.m_blk, q));
                }
            }
        }
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.tma_a);
        tma_prefetch_desc(&p.tma_b);
        tma_prefetch_desc(&p.tma_d);
        if (EPI == 1 && p.c != nullptr) tma_prefetch_desc(&p.tma_c);
    }
    if (warp == 1) {
        tmem_alloc<CG>(s_tmem, Cfg::TMEM_COLS);
        tmem_relinquish<CG>();
    }
    // Everything above touches only this CTA's shared memory, TMEM and the
    // kernel parameters; global memory (operands, scales, metadata, status,
    // split-K scratch) is read or written only after the grids this launch
    // depends on have completed. The next launch in the stream may be
    // scheduled right away (it waits for this grid in turn).
    griddep_launch_dependents();
    griddep_wait();
    if constexpr (KIND == kMasked) {
        // masked_m clamped to [0, max_m]
        for (int g = threadIdx.x; g < p.groups; g += NUM_THREADS) s_mm[g] = min(max(__ldg(p.meta + g), 0), p.rows);
        __syncthreads();
    }
    if constexpr (KIND == kPsum) {
        // first row of every group: s_mm[0] = 0, s_mm[g + 1] = end of group g =
        // min(max(0, psum_m[0..g]), M_total), a running max so that no row
        // belongs to two groups (warp 0: per-lane maxima, then a max-scan)
        if (warp == 0) {
            const int per = (p.groups + 31) / 32;
            const int g0 = static_cast<int>(lane) * per;
            int mx = 0;
            for (int i = 0; i < per; ++i)
                if (g0 + i < p.groups) mx = max(mx, __ldg(p.meta + g0 + i));
            int incl = mx;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= static_cast<uint32_t>(o)) incl = max(incl, v);
            }
            int run = __shfl_up_sync(0xffffffffu, incl, 1);
            if (lane == 0) run = 0;
            for (int i = 0; i < per; ++i) {
                const int g = g0 + i;
                if (g < p.groups) {
                    run = max(run, __ldg(p.meta + g));
                    s_mm[g + 1] = min(run, p.rows);
                }
            }
            if (lane == 0) s_mm[0] = 0;
        }
        __syncthreads();
    }
    if constexpr (KIND == kMasked || KIND == kPsum) {
        // tile prefix over groups (warp 0 scans)
        if (warp == 0) {
            const int per = (p.groups + 31) / 32;
            const int g0 = static_cast<int>(lane) * per;
            int sum = 0;
            for (int i = 0; i < per; ++i) {
                const int g = g0 + i;
                if (g < p.groups) sum += ((group_rows<KIND>(s_mm, g) + BM - 1) / BM) * p.num_n_blocks;
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
                    run += ((group_rows<KIND>(s_mm, g) + BM - 1) / BM) * p.num_n_blocks;
                }
            }
            if (lane == 31) s_prefix[p.groups] = incl;
        }
    }
    if constexpr (KIND == kContiguous) {
        // expert of every 128-row block = largest valid index among its rows
        // (-1: padding only), kept in shared memory when the blocks fit
        // Each warp takes 8 blocks per round (lane l: rows 4l..4l+3 of each,
        // one 16-byte load when m_indices allows) and reduces each block.
        const int nblk = (p.rows + BM - 1) / BM;
        if (nblk <= MAX_CACHED_BLOCKS) {
            constexpr int kWarps = NUM_THREADS / 32;
            const bool vec = (reinterpret_cast<uintptr_t>(p.meta) & 15) == 0;
            auto expert_or_none = [&](int id) { return (id >= 0 && id < p.groups) ? id : -1; };
            for (int b0 = static_cast<int>(warp) * 8; b0 < nblk; b0 += kWarps * 8) {
                int best[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    int m = -1;
                    const int r0 = (b0 + u) * BM + 4 * static_cast<int>(lane);
                    if (b0 + u < nblk) {
                        if (vec && r0 + 3 < p.rows) {
                            const int4 v = __ldg(reinterpret_cast<const int4*>(p.meta + r0));
                            m = max(max(expert_or_none(v.x), expert_or_none(v.y)),
                                    max(expert_or_none(v.z), expert_or_none(v.w)));
                        } else {
                            for (int j = 0; j < 4; ++j)
                                if (r0 + j < p.rows) m = max(m, expert_or_none(__ldg(p.meta + r0 + j)));
                        }
                    }
                    best[u] = m;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int m = __reduce_max_sync(0xffffffffu, best[u]);
                    if (lane == 0 && b0 + u < nblk) s_bexp[b0 + u] = m;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    // every CTA's barriers exist before any cross-CTA signal (pairs, cluster split-K)
    if (CG == 2 || (KIND == kDense && p.split_mode == SPLIT_CLUSTER)) cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int kg_count = (p.kb + 3) / 4;
    const int my_rows = BM * static_cast<int>(rank);  // this CTA's rows inside a tile

    if (warp == 0) {
        // -------------------------------------------------------- TMA producer --
        [[maybe_unused]] uint32_t full_leader0 = 0;  // the leader's stage barriers (pairs)
        if constexpr (CG == 2) full_leader0 = mapa_shared(smem_u32(&full_bar[0]), 0);
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        int gcur = 0;
        Tile cur;
        bool aborted = false;
        for (int t = unit; !aborted && next_tile<KIND, true, CG>(p, s_prefix, s_mm, t, units, gcur, cur, lane);
             t += units) {
            const int a_row = (KIND == kPsum ? cur.row0 : cur.m_blk * BM * CG) + my_rows;
            const int b_row = cur.n_blk * BN + Cfg::B_ROWS * static_cast<int>(rank);
            const int g = max(cur.g, 0);
            for (int gi = cur.kg0; gi < cur.kg1 && !aborted; ++gi) {
            const int kgrp = rot_group(p, t, gi, kg_count);
            for (int kb = 4 * kgrp; kb < min(4 * kgrp + 4, p.kb); ++kb) {
                // the first STAGES slots are free from the start: no wait
                if (issued >= STAGES && !wait_warp(&empty_bar[stage], phase ^ 1u, p, s_abort)) { aborted = true; break; }
                if (elect_one()) {
                    uint8_t* a_dst = smem_a + stage * Cfg::A_BYTES;
                    uint8_t* b_dst = smem_b + stage * Cfg::B_BYTES;
                    const int kx = kb * Cfg::K_PER_STAGE;  // TMA coordinates are in elements
                    if constexpr (CG == 1) {
                        mbar_arrive_expect_tx(&full_bar[stage], Cfg::TX_BYTES);
                        if constexpr (KIND == kMasked) {
                            tma_load_3d(a_dst, &p.tma_a, &full_bar[stage], kx, a_row, cur.g);
                        } else if constexpr (kMnA) {
                            tma_load_2d(a_dst, &p.tma_a, &full_bar[stage], a_row, kx);   // {M, K} box
                        } else {
                            tma_load_2d(a_dst, &p.tma_a, &full_bar[stage], kx, a_row);
                        }
                        if constexpr (kMnB) {
#pragma unroll
                            for (int at = 0; at < BN / 128; ++at)                          // {N, K} boxes
                                tma_load_2d(b_dst + at * kMnAtomBytes, &p.tma_b, &full_bar[stage], b_row + 128 * at, kx);
                        } else if constexpr (KIND == kDense) {
                            tma_load_2d(b_dst, &p.tma_b, &full_bar[stage], kx, b_row);
                        } else {
                            tma_load_3d(b_dst, &p.tma_b, &full_bar[stage], kx, b_row, g);
                        }
                    } else {
                        // the leader arms its barrier for both CTAs' bytes; both
                        // CTAs' loads complete on the leader's barrier. An
                        // MN-major operand is one 128-byte atom per CTA: {M or
                        // N, K} box coordinates.
                        if (leader) mbar_arrive_expect_tx(&full_bar[stage], Cfg::TX_BYTES);
                        const uint32_t fb = full_leader0 + 8u * static_cast<uint32_t>(stage);
                        if constexpr (kMnA) tma_load_2d_pair(a_dst, &p.tma_a, fb, a_row, kx);
                        else tma_load_2d_pair(a_dst, &p.tma_a, fb, kx, a_row);
                        if constexpr (kMnB) {
                            tma_load_2d_pair(b_dst, &p.tma_b, fb, b_row, kx);
                        } else if constexpr (KIND == kDense) {
                            tma_load_2d_pair(b_dst, &p.tma_b, fb, kx, b_row);
                        } else {
                            tma_load_3d_pair(b_dst, &p.tma_b, fb, kx, b_row, g);
                        }
                    }
                }
                __syncwarp();
                ++issued;
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            }
        }
        if (aborted) {
            // let the loads already issued land before shared memory goes away
            if constexpr (CG == 1) {
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < STAGES && i < issued; ++i) {
                    if (--s < 0) { s = STAGES - 1; ph ^= 1u; }
                    wait_quiet(&full_bar[s], ph, p.wait_limit_ns / 16);
                }
            } else {
                sleep_ns(p.wait_limit_ns / 16);  // completion lands on the leader's barrier
            }
        }
    } else if (warp == 6) {
        // ------------------------------------------------------ scale producer --
        // For a pair the leader's warp gathers the words of both CTAs and writes
        // the peer's share into the peer's shared memory, so the hand-off to the
        // MMA warp stays inside the leader CTA; the peer's warp has no work.
        if (DT == kE4M3 && (CG == 1 || leader)) {
            [[maybe_unused]] uint32_t peer_sf0 = 0;  // the peer's scale ring (pairs)
            if constexpr (CG == 2) peer_sf0 = mapa_shared(smem_u32(smem_sf), 1);
            // Groups are visited in the MMA warp's order (tile by tile, K groups
            // in order). Two register sets keep the loads of two groups in
            // flight while a third is stored.
            int ct = unit, cg_cur = 0;
            Tile ctile;
            bool cok = next_tile<KIND, true, CG>(p, s_prefix, s_mm, ct, units, cg_cur, ctile, lane);
            int ckg = cok ? ctile.kg0 : 0;
            auto load_next = [&](ScaleWords<BN, KIND, CG>& w) -> bool {
                if (!cok) return false;
                w.load(p, KIND == kPsum ? ctile.row0 : ctile.m_blk * BM * CG, ctile.n_blk * BN, ctile.g,
                       rot_group(p, ct, ckg, kg_count), lane);
                if (++ckg == ctile.kg1) {
                    ct += units;
                    cok = next_tile<KIND, true, CG>(p, s_prefix, s_mm, ct, units, cg_cur, ctile, lane);
                    if (cok) ckg = ctile.kg0;
                }
                return true;
            };
            int slot = 0;
            uint32_t sf_phase = 0;
            int groups_done = 0;
            // store one group into the next ring slot and publish it; false on abort
            auto put = [&](const ScaleWords<BN, KIND, CG>& w) -> bool {
                if (!wait_warp(&sf_empty_bar[slot], sf_phase ^ 1u, p, s_abort)) return false;
                uint8_t* sfa_slot = smem_sf + slot * Cfg::SF_SLOT_BYTES;
                w.store(sfa_slot, sfa_slot + Cfg::SFA_BYTES, lane);
                if constexpr (CG == 2) {
                    const uint32_t peer_slot = peer_sf0 + static_cast<uint32_t>(slot * Cfg::SF_SLOT_BYTES);
                    w.store_peer(peer_slot, peer_slot + Cfg::SFA_BYTES, lane);
                    fence_proxy_async_cluster();  // remote generic stores -> the async proxy (tcgen05.cp)
                } else {
                    fence_proxy_async_smem();
                }
                __syncwarp();
                // test hook: CTA 0 withholds the arrive of its first group
                const bool withhold = p.test_mode == 1 && blockIdx.x == 0 && groups_done == 0;
                if (lane == 0 && !withhold) mbar_arrive(&sf_full_bar[slot]);
                __syncwarp();
                ++groups_done;
                if (++slot == SF_RING) { slot = 0; sf_phase ^= 1u; }
                return true;
            };
            if (p.sf_vec4) {
                // 16-byte rows of scale words (K groups in order, no rotation):
                // quads of four groups are walked tile by tile, each serving
                // the groups of its tile that it covers; the loads of the next
                // quad are in flight while the current one is stored
                int q_base = cok ? (ctile.kg0 & ~3) : 0;
                auto load_quad = [&](ScaleQuads<BN, KIND, CG>& q) -> bool {
                    if (!cok) return false;
                    q.lo = max(q_base, ctile.kg0);
                    q.hi = min(q_base + 4, ctile.kg1);
                    q.load(p, KIND == kPsum ? ctile.row0 : ctile.m_blk * BM * CG, ctile.n_blk * BN, ctile.g, q_base,
                           lane);
                    q_base += 4;
                    if (q_base >= ctile.kg1) {
                        ct += units;
                        cok = next_tile<KIND, true, CG>(p, s_prefix, s_mm, ct, units, cg_cur, ctile, lane);
                        if (cok) q_base = ctile.kg0 & ~3;
                    }
                    return true;
                };
                auto put_quad = [&](const ScaleQuads<BN, KIND, CG>& q) -> bool {
                    for (int kg = q.lo; kg < q.hi; ++kg) {
                        ScaleWords<BN, KIND, CG> w;
                        q.words(p, w, kg & 3, kg, lane);
                        if (!put(w)) return false;
                    }
                    return true;
                };
                ScaleQuads<BN, KIND, CG> q0, q1;
                bool h0 = load_quad(q0);
                bool h1 = load_quad(q1);
                while (h0) {
                    if (!put_quad(q0)) break;
                    h0 = load_quad(q0);
                    if (!h1) break;
                    if (!put_quad(q1)) break;
                    h1 = load_quad(q1);
                }
            } else {
                ScaleWords<BN, KIND, CG> w0, w1;
                bool v0 = load_next(w0);
                bool v1 = load_next(w1);
                while (v0) {
                    if (!put(w0)) break;
                    v0 = load_next(w0);
                    if (!v1) break;
                    if (!put(w1)) break;
                    v1 = load_next(w1);
                }
            }
        }
    } else if (warp == 1) {
        // ----------------------------------------------------------------- MMA --
        // The whole warp runs the loop and waits by vote; one lane, chosen by
        // elect.sync, issues each batch of tcgen05.mma / cp / commit. Issuing
        // from a converged warp keeps the tensor pipe fed: a loop run by a
        // single lane (or guarded by a lane test) issues the same MMAs about a
        // fifth slower per K-block on this part, because each barrier probe
        // then stalls the issue of the MMAs that follow it.
        if (leader) {
            int stage = 0;
            uint32_t phase = 0;
            int slot = 0;
            uint32_t sf_phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            int gcur = 0;
            Tile c;
            bool aborted = false;
            // Two sets of scale columns: `sf_cur` feeds the MMAs of the current
            // group; the next group's words are copied into `sf_nxt` right after
            // the current group's first K-block is issued, so that wait and
            // copy overlap MMAs already queued (the tensor pipe runs a thread's
            // copies and MMAs in issue order).
            uint32_t sf_cur = tmem_base + Cfg::SF_SET0;
            uint32_t sf_nxt = tmem_base + Cfg::SF_SET1;
            // next group's scale words (both CTAs of a pair) -> TMEM at `dst`;
            // the ring slot is free again once the copy has completed
            auto copy_scales = [&](uint32_t dst) -> bool {
                if constexpr (DT != kE4M3) return true;  // plain BF16 operands carry no scales
                if (!wait_warp(&sf_full_bar[slot], sf_phase, p, s_abort)) return false;
                tc_fence_after();
                if (elect_one()) {
                    const uint8_t* sf_slot = smem_sf + slot * Cfg::SF_SLOT_BYTES;
                    tc_cp_32x128b_warpx4<CG>(dst, smem_desc_sf(smem_u32(sf_slot)));
#pragma unroll
                    for (int ch = 0; ch < Cfg::SFB_CHUNKS; ++ch)
                        tc_cp_32x128b_warpx4<CG>(dst + 4 + 4 * ch,
                                                 smem_desc_sf(smem_u32(sf_slot + Cfg::SFA_BYTES + 512 * ch)));
                    tc_commit<CG>(&sf_empty_bar[slot]);
                }
                __syncwarp();
                if (++slot == SF_RING) { slot = 0; sf_phase ^= 1u; }
                return true;
            };
            for (int t = unit; !aborted && next_tile<KIND, CG == 2, CG>(p, s_prefix, s_mm, t, units, gcur, c, lane);
                 t += units) {
                if (!wait_warp(&tempty_bar[acc], acc_phase ^ 1u, p, s_abort)) { aborted = true; break; }
                tc_fence_after();  // the epilogue's TMEM reads precede the MMAs below
                const uint32_t d_tmem = tmem_base + acc * Cfg::ACC_STRIDE;
                // the tile's first group: its scales go to the set the previous
                // group did not use
                if (!copy_scales(sf_nxt)) { aborted = true; break; }
                {
                    const uint32_t tmp = sf_cur;
                    sf_cur = sf_nxt;
                    sf_nxt = tmp;
                }
                for (int gi = c.kg0; gi < c.kg1 && !aborted; ++gi) {
                    const int kgrp = rot_group(p, t, gi, kg_count);
                    const int kb0 = 4 * kgrp;
                    for (int kb = kb0; kb < min(kb0 + 4, p.kb); ++kb) {
                        // TMA bytes observed complete on the barrier are visible to
                        // the tensor core's shared-memory reads: no fence needed here
                        if (!wait_warp(&full_bar[stage], phase, p, s_abort)) { aborted = true; break; }
                        const uint32_t sf_id = static_cast<uint32_t>(kb & 3);
                        const uint32_t idesc = idesc_with_sf_id(kIdesc, sf_id);
                        const uint32_t sfa_t = sf_cur | (sf_id << 30);
                        const uint32_t sfb_t = (sf_cur + 4) | (sf_id << 30);
                        const uint64_t adesc =
                            kMnA ? smem_desc_sw128_mn(smem_u32(smem_a + stage * Cfg::A_BYTES), kMnLbo, kMnSbo)
                                 : smem_desc_sw128(smem_u32(smem_a + stage * Cfg::A_BYTES));
                        const uint64_t bdesc =
                            kMnB ? smem_desc_sw128_mn(smem_u32(smem_b + stage * Cfg::B_BYTES), kMnLbo, kMnSbo)
                                 : smem_desc_sw128(smem_u32(smem_b + stage * Cfg::B_BYTES));
                        if (elect_one()) {
                            // four MMAs per 128-byte row of K: E4M3 K = 32, BF16 K = 16 per instruction;
                            // each advances the start address by 32 bytes inside the swizzled row
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                // K-major: the next 32 bytes of K in each swizzled row;
                                // MN-major: the next 32 K-rows (4 groups of 8 rows of 128 bytes)
                                const uint64_t koff = static_cast<uint64_t>((k * 32) >> 4);
                                const uint64_t koff_mn = static_cast<uint64_t>((k * 32 * 128) >> 4);
                                const uint32_t accumulate = (gi > c.kg0 || kb > kb0 || k > 0) ? 1u : 0u;
                                if constexpr (DT == kE4M3)
                                    tc_mma_mxf8f6f4_block_scale<CG>(d_tmem, adesc + (kMnA ? koff_mn : koff),
                                                                    bdesc + (kMnB ? koff_mn : koff), idesc, sfa_t,
                                                                    sfb_t, accumulate);
                                else
                                    tc_mma_f16<CG>(d_tmem, adesc + koff, bdesc + koff, Cfg::IDESC, accumulate);
                            }
                            tc_commit<CG>(&empty_bar[stage]);
                        }
                        __syncwarp();
                        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                        if (kb == kb0 && gi + 1 < c.kg1 && !copy_scales(sf_nxt)) { aborted = true; break; }
                    }
                    if (gi + 1 < c.kg1) {
                        const uint32_t tmp = sf_cur;
                        sf_cur = sf_nxt;
                        sf_nxt = tmp;
                    }
                }
                if (aborted) break;
                if (elect_one()) tc_commit<CG>(&tfull_bar[acc]);
                __syncwarp();
                if (++acc == NUM_ACC) { acc = 0; acc_phase ^= 1u; }
            }
            // all MMAs must finish before TMEM is released (in both CTAs)
            if (elect_one()) tc_commit<CG>(drain_bar);
            __syncwarp();
        }
        wait_quiet(drain_bar, 0, p.wait_limit_ns);
    } else {
        // ------------------------------------------------------------ epilogue --
        // Each warp owns 32 rows (its TMEM sub-partition). Per tile it reads
        // the accumulator in batches of up to 128 columns, hands TMEM back to
        // the MMA warp right after the last read, and then writes bf16:
        // 32x32 chunks staged in swizzled shared memory and stored with TMA
        // when all 32 rows may be written, predicated 16-byte stores otherwise.
        // D = C + A.B^T (dense) moves C in and D out through the same staging
        // buffers with TMA (row-wise 16-byte loads and stores of 32 rows at a
        // time measured 10-19% slower on 4096x7168x16384: their many small
        // requests slow the operand loads of the tile being computed).
        const int q = static_cast<int>(warp & 3);   // TMEM sub-partition of this warp
        uint8_t* stg = smem_epi + (warp - 2) * Cfg::EPI_WARP_BYTES;
        [[maybe_unused]] uint32_t tempty_leader0 = 0;  // the leader's accumulator barriers (pairs)
        if constexpr (CG == 2) tempty_leader0 = mapa_shared(smem_u32(&tempty_bar[0]), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        uint32_t epi_phase = 0;
        int gcur = 0;
        int buf = 0;
        [[maybe_unused]] uint32_t c_phase = 0;   // D = C + A.B^T: parity of this warp's C barrier
        bool e_abort = false;                     // a wait inside a chunk's output gave up
        Tile c;
        for (int t = unit; next_tile<KIND, true, CG>(p, s_prefix, s_mm, t, units, gcur, c, lane); t += units) {
            const int row_coord = c.m_blk * BM * CG + my_rows + 32 * q;
            const int mloc = row_coord + static_cast<int>(lane);
            bool valid;
            size_t out_row;
            if constexpr (KIND == kDense) {
                valid = mloc < p.rows;
                out_row = static_cast<size_t>(mloc);
            } else if constexpr (KIND == kMasked) {
                valid = mloc < s_mm[c.g];
                out_row = static_cast<size_t>(c.g) * p.rows + mloc;
            } else if constexpr (KIND == kPsum) {
                valid = mloc < group_rows<kPsum>(s_mm, c.g);   // mloc counts from the group's first row
                out_row = static_cast<size_t>(s_mm[c.g] + mloc);
            } else {
                const int id = (mloc < p.rows) ? __ldg(p.meta + mloc) : -1;
                const bool in_range = id >= 0 && id < p.groups;
                valid = in_range && id == c.g;
                // a 128-row block must hold one expert (rows of a pair's other
                // block may belong to another one, written in the other pass)
                const int own = rank == 0 ? c.e_own[0] : c.e_own[1];
                if (in_range && id != own) atomicOr(p.status, DEVERR_MIXED_EXPERT_BLOCK);
                out_row = static_cast<size_t>(mloc);
            }
            // TMA stores clip at the tensor's edges, so for the dense form rows
            // past M are safe; the grouped forms need every row of the chunk valid.
            const bool use_tma = (KIND == kDense) ? true : (__all_sync(0xffffffffu, valid) != 0);
            if (!wait_warp(&tfull_bar[acc], acc_phase, p, s_abort)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + acc * Cfg::ACC_STRIDE;
            const int n0 = c.n_blk * BN;
            __nv_bfloat16* drow = p.d + out_row * static_cast<size_t>(p.n) + n0;
            constexpr int kMaxBatch = 128;
            constexpr bool kCanSplit = KIND == kDense && CG == 1;
            if constexpr (kCanSplit) {
                if (p.split_mode == SPLIT_CLUSTER) {
                    // split-K inside a cluster: the partials meet in the owners'
                    // shared memory (one tile per CTA, so the ring is free)
                    if (!cluster_split_epilogue<BN, EPI>(p, c, q, warp, lane, taddr, smem_a, red_free, red_full,
                                                         s_abort))
                        break;
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty_bar[acc]);
                    if (++acc == NUM_ACC) { acc = 0; acc_phase ^= 1u; }
                    continue;
                }
            }
            // split-K through global scratch (dense, single CTAs): every unit
            // parks its fp32 partial in the workspace; the unit that finishes a
            // tile last adds the partials in split order (the same sum whichever
            // unit is last) and writes the bf16 tile.
            const bool split = kCanSplit && p.split_mode == SPLIT_SCRATCH;
            bool emit_tile = !split;
            if constexpr (kCanSplit) {
                if (split) {
                    float* part = p.ws + ((static_cast<size_t>(c.base) * p.splits + c.split) * 4 + q) * (BN * 32);
#pragma unroll
                    for (int h = 0; h < BN; h += 128) {
                        const int cols = (BN - h) < kMaxBatch ? (BN - h) : kMaxBatch;
                        uint32_t r[kMaxBatch];
#pragma unroll
                        for (int j = 0; j < kMaxBatch / 32; ++j)
                            if (32 * j < cols) tmem_ld_32x32b_x32(taddr + h + 32 * j, r + 32 * j);
                        tc_wait_ld();
                        if (h + 128 >= BN) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&tempty_bar[acc]);
                        }
                        if (valid) {
#pragma unroll
                            for (int c4 = 0; c4 < kMaxBatch / 4; ++c4)
                                if (4 * c4 < cols)
                                    __stcg(reinterpret_cast<float4*>(part + ((h / 4 + c4) * 32 + lane) * 4),
                                           make_float4(__uint_as_float(r[4 * c4]), __uint_as_float(r[4 * c4 + 1]),
                                                       __uint_as_float(r[4 * c4 + 2]), __uint_as_float(r[4 * c4 + 3])));
                        }
                    }
                    // publish: every thread's partial stores precede the count
                    __threadfence();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(epi_bar);
                    if (!wait_warp(epi_bar, epi_phase, p, s_abort)) break;
                    epi_phase ^= 1u;
                    if (warp == 2 && lane == 0) {
                        const uint32_t done = atomicAdd(&p.counters[c.base], 1u);
                        const bool last = done == static_cast<uint32_t>(p.splits - 1);
                        if (last) atomicExch(&p.counters[c.base], 0u);  // zero again for the next call
                        *s_last = last ? 1 : 0;
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(epi_bar);
                    if (!wait_warp(epi_bar, epi_phase, p, s_abort)) break;
                    epi_phase ^= 1u;
                    emit_tile = *s_last != 0;
                    if (emit_tile) __threadfence();  // the other units' partials are visible from here on
                }
            }
            // fp32 -> bf16 (round to nearest even) of 32 columns starting at tile
            // column hc, written as one 32x32 chunk
            auto emit32 = [&](const uint32_t* v, int hc) {
                const int col = n0 + hc;
                if (col >= p.n || e_abort) return;  // warp-uniform: N tail
                float f[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
                if constexpr (EPI == 1) {
                    // dense form: C comes in and D goes out through the warp's two
                    // 2 KB staging buffers with TMA
                    if (p.out_f32) {
                        // 32 fp32 columns as two boxes of 16 rows x 128 bytes (the
                        // 128-byte swizzle: granule g of row r at g ^ (r & 7)), rows
                        // 0-15 in the first buffer and 16-31 in the second
                        if (lane == 0) bulk_wait_group_read<0>();  // both buffers free
                        __syncwarp();
                        uint8_t* sb = stg + (lane >> 4) * 2048 + (lane & 15) * 128;
                        const uint32_t sw8 = lane & 7u;
                        if (p.c != nullptr) {
                            if (lane == 0) {
                                mbar_arrive_expect_tx(&cbar[q], 4096);
                                tma_load_2d(stg, &p.tma_c, &cbar[q], col, row_coord);
                                tma_load_2d(stg + 2048, &p.tma_c, &cbar[q], col, row_coord + 16);
                            }
                            if (!wait_warp(&cbar[q], c_phase, p, s_abort)) {
                                e_abort = true;
                                return;
                            }
                            c_phase ^= 1u;
#pragma unroll
                            for (int g = 0; g < 8; ++g) {
                                const float4 x = *reinterpret_cast<const float4*>(sb + 16 * (g ^ sw8));
                                f[4 * g] += x.x;
                                f[4 * g + 1] += x.y;
                                f[4 * g + 2] += x.z;
                                f[4 * g + 3] += x.w;
                            }
                        }
#pragma unroll
                        for (int g = 0; g < 8; ++g)
                            *reinterpret_cast<float4*>(sb + 16 * (g ^ sw8)) =
                                make_float4(f[4 * g], f[4 * g + 1], f[4 * g + 2], f[4 * g + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&p.tma_d, stg, col, row_coord);
                            tma_store_2d(&p.tma_d, stg + 2048, col, row_coord + 16);
                            bulk_commit_group();
                        }
                    } else {
                        // bf16: one 32-row x 64-byte box (64-byte swizzle, as below)
                        // per chunk, buffers taken in turn
                        const uint32_t sw = (lane >> 1) & 3u;
                        // the store issued two chunks ago has finished reading this buffer
                        if (lane == 0) bulk_wait_group_read<1>();
                        __syncwarp();
                        uint8_t* sb = stg + buf * 2048;
                        if (p.c != nullptr) {
                            if (lane == 0) {
                                mbar_arrive_expect_tx(&cbar[q], 2048);
                                tma_load_2d(sb, &p.tma_c, &cbar[q], col, row_coord);
                            }
                            if (!wait_warp(&cbar[q], c_phase, p, s_abort)) {
                                e_abort = true;
                                return;
                            }
                            c_phase ^= 1u;
#pragma unroll
                            for (int g = 0; g < 4; ++g) {
                                const uint4 x = *reinterpret_cast<const uint4*>(sb + lane * 64 + 16 * (g ^ sw));
                                const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                                for (int h2 = 0; h2 < 4; ++h2) {
                                    const float2 c2 =
                                        __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[h2]));
                                    f[8 * g + 2 * h2] += c2.x;
                                    f[8 * g + 2 * h2 + 1] += c2.y;
                                }
                            }
                        }
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            uint32_t w4[4];
#pragma unroll
                            for (int h2 = 0; h2 < 4; ++h2) {
                                __nv_bfloat162 b2 = __floats2bfloat162_rn(f[8 * g + 2 * h2], f[8 * g + 2 * h2 + 1]);
                                w4[h2] = *reinterpret_cast<uint32_t*>(&b2);
                            }
                            *reinterpret_cast<uint4*>(sb + lane * 64 + 16 * (g ^ sw)) =
                                make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&p.tma_d, sb, col, row_coord);
                            bulk_commit_group();
                        }
                        buf ^= 1;
                    }
                } else {
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
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
                            else if constexpr (KIND == kPsum) tma_store_2d(&p.tma_d, sb, col, s_mm[c.g] + row_coord);
                            else tma_store_2d(&p.tma_d, sb, col, row_coord);
                            bulk_commit_group();
                        }
                        buf ^= 1;
                    } else if (valid) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            if (col + 8 * q4 < p.n)
                                *reinterpret_cast<uint4*>(drow + hc + 8 * q4) =
                                    make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
                    }
                }
            };
            // the 16-column tail chunk of a 240-wide tile (pairs, dense form):
            // fp32 -> bf16 (or + C, fp32) with direct 16-byte stores of the valid rows
            auto emit16 = [&](const uint32_t* v, int hc) {
                const int col = n0 + hc;
                if (col >= p.n || !valid) return;  // N % 8 == 0: 8-column pieces are wholly in or out
                float f[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) f[i] = __uint_as_float(v[i]);
                const size_t at = out_row * static_cast<size_t>(p.n) + col;
                if constexpr (EPI == 1) {
                    if (p.c != nullptr) {
                        if (p.out_f32) {
                            const float* crow = static_cast<const float*>(p.c) + at;
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4) {
                                if (col + 4 * q4 >= p.n) continue;
                                const float4 x = *reinterpret_cast<const float4*>(crow + 4 * q4);
                                f[4 * q4] += x.x; f[4 * q4 + 1] += x.y; f[4 * q4 + 2] += x.z; f[4 * q4 + 3] += x.w;
                            }
                        } else {
                            const __nv_bfloat16* crow = static_cast<const __nv_bfloat16*>(p.c) + at;
#pragma unroll
                            for (int q8 = 0; q8 < 2; ++q8) {
                                if (col + 8 * q8 >= p.n) continue;
                                const uint4 x = *reinterpret_cast<const uint4*>(crow + 8 * q8);
                                const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                                for (int h2 = 0; h2 < 4; ++h2) {
                                    const float2 c2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[h2]));
                                    f[8 * q8 + 2 * h2] += c2.x;
                                    f[8 * q8 + 2 * h2 + 1] += c2.y;
                                }
                            }
                        }
                    }
                    if (p.out_f32) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            if (col + 4 * q4 < p.n)
                                *reinterpret_cast<float4*>(p.d32 + at + 4 * q4) =
                                    make_float4(f[4 * q4], f[4 * q4 + 1], f[4 * q4 + 2], f[4 * q4 + 3]);
                        return;
                    }
                }
                uint32_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
                    w[i] = *reinterpret_cast<uint32_t*>(&b2);
                }
#pragma unroll
                for (int q8 = 0; q8 < 2; ++q8)
                    if (col + 8 * q8 < p.n)
                        *reinterpret_cast<uint4*>(p.d + at + 8 * q8) =
                            make_uint4(w[4 * q8], w[4 * q8 + 1], w[4 * q8 + 2], w[4 * q8 + 3]);
            };
            if (emit_tile && !(kCanSplit && split)) {
#pragma unroll
                for (int h = 0; h < BN; h += 128) {
                    const int cols = (BN - h) < kMaxBatch ? (BN - h) : kMaxBatch;  // compile-time after unrolling
                    uint32_t r[kMaxBatch];
#pragma unroll
                    for (int j = 0; j < kMaxBatch / 32; ++j) {
                        if (32 * j + 32 <= cols) tmem_ld_32x32b_x32(taddr + h + 32 * j, r + 32 * j);
                        else if (32 * j < cols) tmem_ld_32x32b_x16(taddr + h + 32 * j, r + 32 * j);
                    }
                    tc_wait_ld();
                    if (h + 128 >= BN) {
                        // last TMEM read of this accumulator: hand it back to the MMA warp
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if (CG == 1 || leader) mbar_arrive(&tempty_bar[acc]);
                            else mbar_arrive_cluster(tempty_leader0 + 8u * static_cast<uint32_t>(acc));
                        }
                    }
#pragma unroll
                    for (int j = 0; j < kMaxBatch / 32; ++j) {
                        if (32 * j + 32 <= cols) emit32(r + 32 * j, h + 32 * j);
                        else if (32 * j < cols) emit16(r + 32 * j, h + 32 * j);
                    }
                }
            }
            if constexpr (kCanSplit) {
                if (emit_tile && split) {
                    // this unit finished the tile last: the sum of the partials in
                    // split order, 32 columns at a time, loads of two splits in
                    // flight per round
                    const float* tile_ws = p.ws + (static_cast<size_t>(c.base) * p.splits * 4 + q) * (BN * 32);
                    const size_t split_stride = static_cast<size_t>(4) * BN * 32;
#pragma unroll 1
                    for (int hc = 0; hc < BN; hc += 32) {
                        float acc32[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) acc32[i] = 0.f;
                        if (valid) {
                            const float* src = tile_ws + ((hc / 4) * 32 + lane) * 4;
                            for (int sp0 = 0; sp0 < p.splits; sp0 += 2) {
                                float4 v[2][8];
#pragma unroll
                                for (int u = 0; u < 2; ++u)
                                    if (sp0 + u < p.splits)
#pragma unroll
                                        for (int c4 = 0; c4 < 8; ++c4)
                                            v[u][c4] = __ldcg(reinterpret_cast<const float4*>(
                                                src + (sp0 + u) * split_stride + c4 * 128));
#pragma unroll
                                for (int u = 0; u < 2; ++u)
                                    if (sp0 + u < p.splits)
#pragma unroll
                                        for (int c4 = 0; c4 < 8; ++c4) {
                                            acc32[4 * c4] += v[u][c4].x;
                                            acc32[4 * c4 + 1] += v[u][c4].y;
                                            acc32[4 * c4 + 2] += v[u][c4].z;
                                            acc32[4 * c4 + 3] += v[u][c4].w;
                                        }
                            }
                        }
                        uint32_t bits[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) bits[i] = __float_as_uint(acc32[i]);
                        emit32(bits, hc);
                    }
                }
            }
            if (e_abort) break;
            if (++acc == NUM_ACC) { acc = 0; acc_phase ^= 1u; }
        }
        // a C load whose wait gave up may still land: let it, within a bound,
        // before shared memory goes away
        if (e_abort) wait_quiet(&cbar[q], c_phase, p.wait_limit_ns / 16);
        // every bulk store must have completed before the CTA exits
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    // neither CTA of a pair frees TMEM while the pair still uses it; no CTA of a
    // split-K cluster exits while peers may still write into its shared memory
    if (CG == 2 || (KIND == kDense && p.split_mode == SPLIT_CLUSTER)) cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<CG>(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace dg
