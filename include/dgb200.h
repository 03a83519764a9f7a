/*
 * dgb200 -- FP8 (E4M3) block-scaled GEMMs and the UE8M0 scale pack for B200 (sm_100a).
 *
 * C ABI of libdgb200.so. Every argument is a plain pointer or an integer; no
 * framework type appears here. Device pointers point to memory on the current
 * CUDA device; `stream` is a cudaStream_t passed as void* (NULL = legacy
 * default stream).
 *
 * Operation (dense, contiguous, masked and psum_m GEMM forms): D = A . B^T
 * ("NT"), E4M3 operands, fp32 accumulation, bf16 output, no C term (the
 * C term, fp32 output, other operand layouts and BF16 operands have calls of
 * their own below). Sources: "DeepInside DeepGEMM:
 * Unpacking DeepSeek's Unified Tensor Core Library for SM90 and SM100",
 * section 4 (the standard non-grouped FP8 NT GEMM computes D = C + A @ B.T)
 * and section 2 (on SM100 the scaling factors are UE8M0, four packed into one
 * torch.int).
 *
 * Scales. Activations (A) carry one scale per 1x128 block along K, weights (B)
 * one scale per 128x128 block (the *_sfb_gran calls also take one per 1x128
 * block of each row of B). A scale is a UE8M0 byte e meaning 2^(e-127).
 * Scale rows are packed four bytes per int32, little-endian, consecutive
 * along K: byte j of word i is K-block 4*i + j. With KB = K/128 and
 * KP = ceil(KB/4):
 *     sfa: int32 [rows, KP]            row-major, one row per row of A
 *     sfb: int32 [ceil(N/128), KP]     row-major, one row per 128 rows of B
 * pack_ue8m0() produces exactly this layout from fp32 scales.
 *
 * Layouts. All tensors are dense and row-major. A rows are K bytes long, B rows
 * K bytes, D rows N bf16 values.
 *
 * Ownership. The caller allocates and owns every buffer. The library keeps no
 * per-call state and allocates no device memory, neither in a call nor when it
 * sets up a device: its only device data are static variables of its module
 * (the 4-byte status word below, and the scratch of fp8_gemm_nt_noalloc).
 *
 * Streams. Work goes only on the stream given. Calls are asynchronous and
 * reentrant: calls on different streams (or host threads) may run at the same
 * time, since no compute call except fp8_gemm_nt_noalloc touches memory other
 * than its own arguments and the status word.
 *
 * CUDA Graph capture. Every compute entry point of the method (all but
 * fp8_gemm_nt_noalloc, about which no claim is made) is capture safe: no host
 * synchronisation, no allocation, no host reads of device values, and a launch
 * configuration fixed by the scalar sizes alone ("DeepGEMM CUDA Graph
 * Compatibility for Masked Grouped GEMMs: Implementation Guide", sections
 * Stateless Kernel Architecture and Tensor-Based Metadata Arguments). All
 * variable metadata (masked_m, psum_m, m_indices, scales) is read on the device. The
 * first call on a device configures the kernels (cudaFuncSetAttribute); make
 * it, or dgb200_init(), before capturing.
 *
 * Errors. Host-checkable mistakes return a status without launching anything:
 * null pointers, non-positive sizes, K not a multiple of 128, N not a multiple
 * of 8, misaligned pointers (A, B, D need 16-byte alignment; scales and
 * metadata 4-byte), sizes past the limits below. A failed launch returns
 * DG_ERR_CUDA. Device values are never checked on the host; the kernels
 * clamp them (see each call) and record problems in a device status word that
 * dgb200_device_error() reads. Every wait inside a kernel is bounded: a wait
 * that runs out sets DG_DEVERR_TIMEOUT and the kernel returns instead of
 * hanging.
 *
 * Limits: 1 <= M, N; N % 8 == 0; K % 128 == 0; 128 <= K <= 2^20;
 * rows * K < 2^40 for every operand; G <= 1024 for the masked and psum_m forms.
 */
#ifndef DGB200_H
#define DGB200_H

#include <stdint.h>

#if defined(__GNUC__)
#define DG_API __attribute__((visibility("default")))
#else
#define DG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DG_OK = 0,
    DG_ERR_INVALID_ARG = 1,    /* null pointer, bad size or bad combination */
    DG_ERR_ALIGNMENT = 2,      /* pointer or row pitch not aligned as required */
    DG_ERR_UNSUPPORTED = 3,    /* valid request outside this build's limits */
    DG_ERR_NOT_INITIALIZED = 4,/* no usable CUDA device / driver entry point */
    DG_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed */
    DG_ERR_SCRATCH_TOO_SMALL = 6 /* fp8_gemm_nt_noalloc: the request needs more
                                    scratch than its static arrays hold */
} dg_status;

/* Bits of the device status word (see dgb200_device_error). */
#define DG_DEVERR_TIMEOUT             1u /* a bounded wait inside a kernel ran out */
#define DG_DEVERR_MIXED_EXPERT_BLOCK  2u /* contiguous: an aligned 128-row block held two experts */

/* Human-readable name of a status code (static string). */
DG_API const char* dgb200_status_string(dg_status s);

/*
 * Configure the kernels for CUDA device `device` (an ordinal as in
 * cudaSetDevice): checks that it is an sm_100 part, caches its SM count, sets
 * the kernels' dynamic shared-memory limits and counts how many CTA pairs and
 * clusters fit on it at once. Allocates nothing. The caller's current device
 * is unchanged on return. Idempotent and thread safe. The first compute call
 * on a device does the same implicitly; call this eagerly before any CUDA
 * Graph capture.
 * Returns DG_ERR_INVALID_ARG for an ordinal that names no device,
 * DG_ERR_UNSUPPORTED for a device other than sm_100, DG_ERR_NOT_INITIALIZED
 * when no CUDA driver or device is usable.
 */
DG_API dg_status dgb200_init(int device);

/*
 * Read the device status word of the current device (DG_DEVERR_* bits, 0 when
 * no kernel recorded a problem) into *code (host pointer) and reset it to
 * zero, like cudaGetLastError. Synchronises the device: never call it inside a
 * stream capture.
 */
DG_API dg_status dgb200_last_device_error(int* code);

/*
 * Read the device status word of the current device into *bits (host pointer)
 * and, if clear != 0, reset it to zero. Synchronises the device: never call it
 * inside a stream capture.
 */
DG_API dg_status dgb200_device_error(uint32_t* bits, int clear);

/*
 * Force the N tile width of the GEMM kernels (0 restores the built-in
 * heuristic). Allowed widths: see dgb200_block_n_supported(). Process-wide;
 * meant for tests and tuning.
 */
DG_API dg_status dgb200_set_block_n(int block_n);
DG_API int dgb200_block_n_supported(int block_n);

/*
 * Force the dense and contiguous GEMMs to run on single CTAs (1) or on CTA
 * pairs (2, tcgen05 cta_group::2 with a 256-row tile); 0 restores the
 * heuristic. The masked form always uses single CTAs. Process-wide; meant for
 * tests and tuning.
 * Returns DG_ERR_UNSUPPORTED for other values; a forced combination of tile
 * width and group that is not built makes the GEMM calls return
 * DG_ERR_UNSUPPORTED.
 */
DG_API dg_status dgb200_set_cta_group(int cta_group);

/*
 * Split-K for the dense GEMMs fp8_gemm_nt, fp8_gemm_nt_acc and
 * fp8_gemm_nt_sfb_gran (process-wide; tests and tuning). 0 restores the
 * heuristic, which splits K only when the output tiles alone leave SMs idle
 * (small M). 1 never splits. s >= 2 splits every such call into s ranges of
 * whole K groups (four 128-K blocks each; with G groups, range i covers groups
 * [i*G/s, (i+1)*G/s)); a combination that is not possible (s larger than G, s
 * larger than the tile width / 8, CTA pairs forced) makes the dense call
 * return DG_ERR_UNSUPPORTED.
 * The s units of an output tile run as one thread-block cluster of s CTAs.
 * Each computes the fp32 partial of its K range in tensor memory; the tile's
 * columns are dealt out among the CTAs in 8-column pieces, every CTA sends
 * the pieces it does not own to their owner's shared memory (distributed
 * shared memory), and each owner adds the s partials of its pieces in split
 * order and writes them. No global memory besides D is used, so splitting
 * calls may run concurrently on several streams, and repeated calls give
 * identical bits.
 * Returns DG_ERR_UNSUPPORTED for s outside [0, 8].
 */
DG_API dg_status dgb200_set_splits(int splits);

/*
 * Test hook for the failure path (process-wide). wait_limit_ms bounds every
 * wait inside the GEMM kernels (0 restores the default, 2000 ms). mode 1 makes
 * CTA 0 of each GEMM launch withhold the arrive that publishes its first group
 * of scale words, so a wait runs out: that launch leaves its output incomplete, sets
 * DG_DEVERR_TIMEOUT and returns; the CUDA context stays usable. mode 0 is
 * normal operation.
 */
DG_API dg_status dgb200_set_test_hooks(int mode, int wait_limit_ms);

/*
 * Dense FP8 NT GEMM ("DeepInside DeepGEMM", section 4: fp8_gemm_nt).
 *   a   : device, E4M3 [M, K]
 *   sfa : device, int32 [M, KP]             packed UE8M0, one per 1x128 block
 *   b   : device, E4M3 [N, K]
 *   sfb : device, int32 [ceil(N/128), KP]   packed UE8M0, one per 128x128 block
 *   d   : device, bf16 [M, N]               written completely
 */
DG_API dg_status fp8_gemm_nt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                      void* d, int M, int N, int K, void* stream);

/*
 * Dense FP8 GEMM in the other operand layouts ("DeepInside DeepGEMM", section 2:
 * SM100 supports the NT, TN, NN and TT layouts). D[m, n] = sum_k A[m, k] B[n, k]
 * with scales as in fp8_gemm_nt (sfa [M, KP] by rows of A, sfb [ceil(N/128), KP]
 * by 128-row blocks of B), whatever the storage:
 *   fp8_gemm_nn : a E4M3 [M, K] (K contiguous), b E4M3 [K, N] (N contiguous)
 *   fp8_gemm_tn : a E4M3 [K, M] (M contiguous), b E4M3 [K, N] (N contiguous)
 *   fp8_gemm_tt : a E4M3 [K, M] (M contiguous), b E4M3 [N, K] (K contiguous)
 *   d           : bf16 [M, N]
 * An operand stored M- or N-contiguous is loaded in 128-byte swizzle atoms of
 * that dimension and fed to the MMA as an MN-major operand (no transposition
 * pass). Limits as fp8_gemm_nt, plus M % 16 == 0 when A is stored [K, M] and
 * N % 16 == 0 when B is stored [K, N] (16-byte row pitch). No split-K; N tile
 * 128 or 256 on single CTAs, 256 on CTA pairs (dgb200_set_cta_group).
 */
DG_API dg_status fp8_gemm_nn(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d, int M,
                             int N, int K, void* stream);
DG_API dg_status fp8_gemm_tn(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d, int M,
                             int N, int K, void* stream);
DG_API dg_status fp8_gemm_tt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d, int M,
                             int N, int K, void* stream);

/*
 * Dense FP8 NT GEMM with an accumulation matrix, D = C + A . B^T ("DeepInside
 * DeepGEMM", section 4: the standard non-grouped FP8 NT GEMM computes
 * D = C + A @ B.T and takes the output dtype).
 *   a, sfa, b, sfb : as fp8_gemm_nt
 *   c       : device, [M, N] in D's type (bf16, or fp32 when out_f32 = 1), or
 *             NULL for C = 0. It is added to the fp32 accumulation before the
 *             final conversion. c may equal d (in-place accumulation); it must
 *             not overlap d otherwise. 16-byte aligned.
 *   d       : device, bf16 [M, N] (out_f32 = 0, round to nearest even) or
 *             fp32 [M, N] (out_f32 = 1); written completely.
 * Limits and errors as fp8_gemm_nt; out_f32 outside {0, 1} returns
 * DG_ERR_INVALID_ARG. Same tiling, split-K and capture safety.
 */
DG_API dg_status fp8_gemm_nt_acc(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, const void* c,
                                 void* d, int M, int N, int K, int out_f32, void* stream);

/*
 * fp8_gemm_nt_noalloc: the dense GEMM of fp8_gemm_nt (same arguments, layouts,
 * limits and results) that allocates no device memory, on any call. The pages
 * of the method have no counterpart of this call; it exists for callers that
 * may not allocate (a framework whose caching allocator already holds the
 * device's memory, a server that plans all memory up front and forbids
 * allocation on the request path, code that must not let cudaMalloc/cudaFree
 * synchronise the device).
 *   splits : 0 = the tile model's choice among configurations whose split-K
 *            scratch fits the static arrays below (never DG_ERR_SCRATCH_TOO_SMALL);
 *            1 = no split-K; s >= 2 = exactly s ranges of K groups (as
 *            dgb200_set_splits describes), with the tile width chosen among
 *            those whose partials fit the static arrays.
 * Unlike the other dense calls, the units of a split tile here meet through
 * global scratch, not inside a cluster: each writes its fp32 partial tile to
 * the scratch and the last one to finish adds the partials in split order
 * (the same order as the cluster form, so equal configurations give equal
 * bits). The scratch lives in file-scope __device__ arrays of the library,
 * found with cudaGetSymbolAddress: at most 8 MiB of fp32 partials (2^21
 * floats; a split call needs ceil(M/128) * ceil(N/BN) * s * 128 * BN * 4 bytes
 * for its N tile BN) and 1024 output tiles. A request that no tile width can
 * serve within these limits returns DG_ERR_SCRATCH_TOO_SMALL before any device
 * work;
 * s > 16 returns DG_ERR_UNSUPPORTED. A splitting call first zeroes the tile
 * counters it uses (an asynchronous memset on `stream`).
 * The scratch is shared by every caller of this function on a device: calls
 * that overlap in time (two streams, two host threads, or one call still
 * running when the next one starts on another stream) race on it and give
 * wrong results. Calls on one stream are ordered and safe.
 * The first call on a device does per-device set-up (kernel attributes,
 * symbol addresses; no allocation).
 */
DG_API dg_status fp8_gemm_nt_noalloc(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d,
                                     int M, int N, int K, int splits, void* stream);

/*
 * Contiguous M-grouped FP8 GEMM for MoE ("DeepGEMM tested by Novita AI",
 * grouped GEMM with continuous storage layout, used for training forward and
 * prefill). Rows of A are concatenated by expert; m_indices[r] is the expert
 * of row r, -1 on padding rows.
 *   a         : device, E4M3 [M_total, K]
 *   sfa       : device, int32 [M_total, KP]
 *   b         : device, E4M3 [G, N, K]
 *   sfb       : device, int32 [G, ceil(N/128), KP]
 *   d         : device, bf16 [M_total, N]
 *   m_indices : device, int32 [M_total]
 * Contract: rows form aligned 128-row blocks (rows 128*i .. 128*i+127); within
 * a block every row whose index lies in [0, G) names the same expert. Rows with
 * an index outside [0, G) are padding: they are not computed and their rows of
 * D are left untouched. A block holding two experts computes only the rows of
 * the larger index, leaves the others untouched and sets
 * DG_DEVERR_MIXED_EXPERT_BLOCK.
 */
DG_API dg_status m_grouped_fp8_gemm_nt_contiguous(const void* a, const int32_t* sfa,
                                           const void* b, const int32_t* sfb,
                                           void* d, const int32_t* m_indices,
                                           int M_total, int N, int K, int G, void* stream);

/*
 * Masked M-grouped FP8 GEMM for MoE decode ("DeepGEMM CUDA Graph Compatibility
 * for Masked Grouped GEMMs", Tensor-Based Metadata Arguments: masked_m is a
 * device tensor and max_m_per_group a host integer).
 *   a        : device, E4M3 [G, max_m, K]
 *   sfa      : device, int32 [G, max_m, KP]
 *   b        : device, E4M3 [G, N, K]
 *   sfb      : device, int32 [G, ceil(N/128), KP]
 *   d        : device, bf16 [G, max_m, N]
 *   masked_m : device, int32 [G]; group g uses its first masked_m[g] rows,
 *              clamped on the device to [0, max_m].
 * Rows at or beyond masked_m[g] are never read for output and their rows of D
 * are never written (a pre-filled sentinel survives). The grid depends only on
 * (G, max_m, N, K), so a captured graph can be replayed with new masked_m.
 */
DG_API dg_status m_grouped_fp8_gemm_nt_masked(const void* a, const int32_t* sfa,
                                       const void* b, const int32_t* sfb,
                                       void* d, const int32_t* masked_m,
                                       int G, int max_m, int N, int K, void* stream);

/*
 * M-grouped FP8 GEMM with the groups given by psum_m ("DeepGEMM CUDA Graph
 * Compatibility for Masked Grouped GEMMs", Tensor-Based Metadata Arguments:
 * psum_m is passed as a pre-allocated device tensor; the page gives no
 * definition). Reading: psum_m[g] is the inclusive prefix sum of the groups'
 * row counts, so the rows of all groups lie end to end in A without padding
 * and group g owns rows [psum_m[g-1], psum_m[g]) (psum_m[-1] = 0).
 *   a       : device, E4M3 [M_total, K]
 *   sfa     : device, int32 [M_total, KP]
 *   b       : device, E4M3 [G, N, K]
 *   sfb     : device, int32 [G, ceil(N/128), KP]
 *   d       : device, bf16 [M_total, N]
 *   psum_m  : device, int32 [G], read on the device only.
 * On the device the group ends are clamped to a running maximum in
 * [0, M_total] (end_g = min(max(0, psum_m[0..g]), M_total), start_g =
 * end_{g-1}): a decreasing entry gives an empty group, no row belongs to two
 * groups, and rows in no group (past the last end) are never written.
 * A group may start at any row: a 128-row tile that reaches into the next
 * group computes those rows but writes only its own. Limits as the masked
 * form (G <= 1024); single CTAs. The grid depends only on (M_total, N, K, G),
 * so a captured graph can be replayed with new psum_m.
 */
DG_API dg_status m_grouped_fp8_gemm_nt_psum(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                            void* d, const int32_t* psum_m, int M_total, int N, int K, int G,
                                            void* stream);

/*
 * The three FP8 forms with a choice of B-scale granularity ("DeepInside
 * DeepGEMM", section 4: the minimal FP8 GEMM example gives the right-hand
 * operand one scale row per row, b_sf of shape [n, k / 128]).
 *   sfb_gran_n : rows of B that share one packed scale row:
 *                128 -> 128x128 blocks, sfb as in the calls above
 *                       ([ceil(N/128), KP] per weight matrix);
 *                1   -> 1x128 blocks, sfb int32 [N, KP] per weight matrix
 *                       ([G, N, KP] for the grouped forms), row n of B scaled
 *                       by byte (k / 128) % 4 of word (k / 128) / 4 of row n.
 *                Any other value returns DG_ERR_INVALID_ARG without launching.
 * Every other argument, limit, error and property (capture safety, untouched
 * rows, split-K for the dense form) is that of fp8_gemm_nt_acc,
 * m_grouped_fp8_gemm_nt_contiguous and m_grouped_fp8_gemm_nt_masked; with
 * sfb_gran_n = 128 the results are identical to theirs. The scale rows are
 * read by the scale-producer warp only, so the tile schedule and the main
 * loop are unchanged.
 */
DG_API dg_status fp8_gemm_nt_sfb_gran(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                      int sfb_gran_n, const void* c, void* d, int M, int N, int K, int out_f32,
                                      void* stream);
DG_API dg_status m_grouped_fp8_gemm_nt_contiguous_sfb_gran(const void* a, const int32_t* sfa, const void* b,
                                                           const int32_t* sfb, int sfb_gran_n, void* d,
                                                           const int32_t* m_indices, int M_total, int N, int K, int G,
                                                           void* stream);
DG_API dg_status m_grouped_fp8_gemm_nt_masked_sfb_gran(const void* a, const int32_t* sfa, const void* b,
                                                       const int32_t* sfb, int sfb_gran_n, void* d,
                                                       const int32_t* masked_m, int G, int max_m, int N, int K,
                                                       void* stream);

/*
 * Masked M-grouped BF16 GEMM ("DeepGEMM CUDA Graph Compatibility for Masked
 * Grouped GEMMs", Core Components: the BF16 masked grouped GEMM kernel, and
 * Tensor-Based Metadata Arguments). Plain bf16 operands, no scales; fp32
 * accumulation, bf16 output.
 *   a        : device, bf16 [G, max_m, K]
 *   b        : device, bf16 [G, N, K]
 *   d        : device, bf16 [G, max_m, N]
 *   masked_m : device, int32 [G]; group g uses its first masked_m[g] rows,
 *              clamped on the device to [0, max_m].
 * Limits: K % 64 == 0 (one 128-byte row of K per pipeline stage), N % 8 == 0,
 * G <= 1024, a / b / d 16-byte aligned. Rows at or beyond masked_m[g] are never
 * written (a pre-filled sentinel survives). The grid depends only on
 * (G, max_m, N, K); the call is capture safe like the FP8 masked GEMM.
 */
DG_API dg_status m_grouped_bf16_gemm_nt_masked(const void* a, const void* b, void* d, const int32_t* masked_m, int G,
                                               int max_m, int N, int K, void* stream);

/*
 * Capture-safe UE8M0 pack ("[GH-ISSUE #414] pack_ue8m0_to_int is not CUDA Graph
 * capture safe", Expected behavior). For fp32 scales sf [rows, cols] writes
 * packed [rows, ceil(cols/4)] int32 with byte (bits(sf[r][c]) >> 23) & 0xFF at
 * byte c % 4 of word c / 4 (zero bytes complete the last word). No value
 * checks: a scale that is not a positive power of two packs to its exponent
 * field. Both pointers are device pointers, 4-byte aligned.
 */
DG_API dg_status pack_ue8m0(const float* sf, int32_t* packed, int64_t rows, int cols, void* stream);

/*
 * Optional validation of the same scales, kept off the pack path as the issue
 * asks: writes to *bad_count (device int32) the number of entries whose sign
 * bit is set or whose mantissa is non-zero. Capture safe (the result stays on
 * the device).
 */
DG_API dg_status pack_ue8m0_validate(const float* sf, int64_t rows, int cols, int32_t* bad_count, void* stream);

/*
 * Per-token FP8 quantiser with UE8M0 block scales ("DeepInside DeepGEMM",
 * section 5 Production Gotchas: the FP8 cast of the activations and the
 * packing of their scales go in a dedicated kernel before the GEMM). Produces
 * the A operand of the GEMMs above in one pass.
 *   x         : device, [rows, K] bf16 (x_f32 = 0) or fp32 (x_f32 = 1)
 *   q         : device, E4M3 [rows, K] (written completely)
 *   sf_packed : device, int32 [rows, ceil(K/512)]: the UE8M0 scale of every
 *               1x128 block, four per word (byte j of word i = block 4i + j,
 *               unused bytes of the last word zero), as pack_ue8m0 writes them
 *   sf_f32    : device, fp32 [rows, K/128] (the same scales as floats), or NULL
 * Per 1x128 block: amax = max(max |x|, 1e-4), scale 2^e with
 * e = ceil(log2(amax / 448)), codes = E4M3(x / 2^e) rounded to nearest even.
 * Limits: K % 128 == 0; x and q 16-byte aligned. Values must be finite (NaN or
 * infinity give unspecified codes). Capture safe; reads nothing back.
 */
DG_API dg_status quantize_fp8_1x128(const void* x, int x_f32, void* q, int32_t* sf_packed, float* sf_f32,
                                    int64_t rows, int K, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DGB200_H */
