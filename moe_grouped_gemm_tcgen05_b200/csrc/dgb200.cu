// Host side of libdgb200.so: the C ABI declared in include/dgb200.h.
//
// Each compute call validates its scalars and pointers on the host, encodes
// the TMA tensor maps (driver entry point, no libcuda link), picks a tile
// width from the sizes and the SM count, and launches one kernel on the
// caller's stream. A compute call allocates nothing, never synchronises and
// reads no device value, so the calls of the method can be captured in a CUDA
// Graph (no claim is made for fp8_gemm_nt_noalloc). The library
// allocates no device memory at all: split-K adds its partial tiles inside a
// thread-block cluster (distributed shared memory), and the device status word
// and the scratch of fp8_gemm_nt_noalloc are static __device__ variables.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "dgb200.h"
#include "gemm_kernel.cuh"
#include "pack_kernel.cuh"

// Device status word (DG_DEVERR_* bits). One per device that loads the library.
__device__ uint32_t g_dg_device_status = 0;

// Split-K scratch of fp8_gemm_nt_noalloc, part of the module image instead of
// an allocation. Some callers may not allocate device memory at all: a
// framework whose caching allocator has already reserved the device's memory
// (a library cudaMalloc then fails, or fragments the pool behind its back), a
// server that plans every byte up front and treats an allocation on the
// request path as a latency spike and an out-of-memory risk, or code running
// where cudaMalloc / cudaFree would synchronise the device at a bad moment.
// These arrays exist as soon as the module is loaded; calls find them with
// cudaGetSymbolAddress. Limits: 8 MiB of fp32 partials, 1024 output tiles.
constexpr size_t kStaticPartialFloats = size_t(2) << 20;
constexpr int kStaticCounters = 1024;
static __device__ __align__(256) float g_noalloc_partials[kStaticPartialFloats];
static __device__ __align__(256) uint32_t g_noalloc_counters[kStaticCounters];

namespace {

using dg::GemmParams;

constexpr int kMaxDevices = 64;
constexpr int kMaxClusterSplits = dg::MAX_CLUSTER_SPLITS;

struct DeviceState {
    std::atomic<bool> ready{false};  // set (release) once every field below is filled
    int sms = 0;
    uint32_t* status = nullptr;  // address of g_dg_device_status on this device
    int max_pairs[80] = {};      // co-resident CTA pairs per kernel entry (cluster kernels only)
    // co-resident clusters of s CTAs (s = 2..8) per kernel entry, for the
    // cluster split-K of the dense single-CTA kernels (0: not launchable)
    int max_clusters[80][kMaxClusterSplits + 1] = {};
    // fp8_gemm_nt_noalloc only: split-K scratch in the library's static arrays
    float* split_ws = nullptr;
    uint32_t* split_counters = nullptr;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
// Per-device state of fp8_gemm_nt_noalloc: the same set-up without the
// workspace allocation; split_ws / split_counters point at the static arrays.
DeviceState g_dev_noalloc[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::atomic<int> g_force_bn{0};
std::atomic<int> g_force_cg{0};
std::atomic<int> g_force_splits{0};
std::atomic<int> g_test_mode{0};
std::atomic<uint64_t> g_wait_limit_ns{dg::DEFAULT_WAIT_LIMIT_NS};
// DGB200_LOG=1 in the environment prints each GEMM launch's configuration to stderr.
const bool g_log = [] {
    const char* v = std::getenv("DGB200_LOG");
    return v != nullptr && v[0] == '1';
}();
// Kernels are launched with programmatic stream serialization: a launch may
// start while the previous kernel in the stream drains; each kernel waits for
// it (griddepcontrol.wait) before touching global memory. DGB200_PDL=0 turns
// this off (plain stream order).
const bool g_pdl = [] {
    const char* v = std::getenv("DGB200_PDL");
    return !(v != nullptr && v[0] == '0');
}();
// DGB200_K_ROTATE=1 makes every tile start its K walk at a rotated group (default: in order).
const int g_k_rotate = [] {
    const char* v = std::getenv("DGB200_K_ROTATE");
    return (v != nullptr && v[0] == '1') ? 1 : 0;
}();
// Scale rows whose length is a multiple of 4 words, on 16-byte aligned bases,
// are read 16 bytes (four K groups) per row at a time when the K groups are
// walked in order: A's rows always (dense form), B's rows when B is scaled per
// row (every form); with 128x128 B blocks, B's broadcast words are read per
// group. DGB200_SF_VEC4=0 reads one word per row and group instead. Measured
// on 4096x7168x16384 (BN 224, CTA pairs; the leader reads the scale rows of
// 256 rows of A, which do not stay in L1 between groups): 316 -> 308 us with
// 128x128 B blocks, 384 -> 359 us with per-row B scales. (Reading B's
// broadcast words 16 bytes at a time too measured slower, 325 vs 311 us.)
const bool g_sf_vec4 = [] {
    const char* v = std::getenv("DGB200_SF_VEC4");
    return !(v != nullptr && v[0] == '0');
}();

// --------------------------------------------------------------- kernels ----

template <int BN, int KIND, int CG, int DT, int LAYOUT = 0, int EPI = 0, int AR = dg::BM>
void* kernel_ptr() {
    return reinterpret_cast<void*>(&dg::fp8_block_scaled_gemm_kernel<BN, KIND, CG, DT, LAYOUT, EPI, AR>);
}

struct KernelEntry {
    int bn;
    int kind;
    int cg;      // CTAs per MMA unit (1, or a cluster pair)
    int dt;      // operand type (dg::kE4M3 block-scaled, dg::kBF16)
    int layout;  // dense: bit 0 A stored [K, M], bit 1 B stored [K, N]
    int epi;     // dense: 1 = epilogue of D = C + A.B^T (bf16 or fp32 D)
    int a_rows;  // rows of A per stage: 128, or 64 (dense, M <= 64)
    void* fn;
    int smem;
    int stages;       // depth of the operand ring
    int stage_bytes;  // bytes of one stage (A and B tiles)
};

#define DG_ENTRY_TLEA(BN, KIND, CG, DT, LAYOUT, EPI, AR)                                                        \
    {BN, KIND, CG, DT, LAYOUT, EPI, AR, kernel_ptr<BN, KIND, CG, DT, LAYOUT, EPI, AR>(),                        \
     dg::GemmConfig<BN, CG, dg::sched_ints<KIND>(), DT, AR>::SMEM_BYTES,                                          \
     dg::GemmConfig<BN, CG, dg::sched_ints<KIND>(), DT, AR>::STAGES,                                              \
     dg::GemmConfig<BN, CG, dg::sched_ints<KIND>(), DT, AR>::STAGE_BYTES}
#define DG_ENTRY_TLE(BN, KIND, CG, DT, LAYOUT, EPI) DG_ENTRY_TLEA(BN, KIND, CG, DT, LAYOUT, EPI, dg::BM)
#define DG_SMALL_A(BN) DG_ENTRY_TLEA(BN, dg::kDense, 1, dg::kE4M3, 0, 0, 64)
#define DG_ENTRY_TL(BN, KIND, CG, DT, LAYOUT) DG_ENTRY_TLE(BN, KIND, CG, DT, LAYOUT, 0)
#define DG_ENTRY_T(BN, KIND, CG, DT) DG_ENTRY_TL(BN, KIND, CG, DT, 0)
#define DG_ACC(BN, CG) DG_ENTRY_TLE(BN, dg::kDense, CG, dg::kE4M3, 0, 1)
#define DG_LAYOUT(BN, LAYOUT) DG_ENTRY_TL(BN, dg::kDense, 1, dg::kE4M3, LAYOUT)
#define DG_LAYOUT_PAIR(BN, LAYOUT) DG_ENTRY_TL(BN, dg::kDense, 2, dg::kE4M3, LAYOUT)
#define DG_ENTRY(BN, KIND, CG) DG_ENTRY_T(BN, KIND, CG, dg::kE4M3)
#define DG_BF16_MASKED(BN) DG_ENTRY_T(BN, dg::kMasked, 1, dg::kBF16)
#define DG_ALL_KINDS(BN) \
    DG_ENTRY(BN, dg::kDense, 1), DG_ENTRY(BN, dg::kContiguous, 1), DG_ENTRY(BN, dg::kMasked, 1), DG_ENTRY(BN, dg::kPsum, 1)

const KernelEntry kKernels[] = {
    DG_ALL_KINDS(64),  DG_ALL_KINDS(96),  DG_ALL_KINDS(128), DG_ALL_KINDS(160),
    DG_ALL_KINDS(192), DG_ALL_KINDS(224), DG_ALL_KINDS(256),
    DG_ENTRY(128, dg::kDense, 2), DG_ENTRY(160, dg::kDense, 2), DG_ENTRY(192, dg::kDense, 2),
    DG_ENTRY(224, dg::kDense, 2), DG_ENTRY(240, dg::kDense, 2), DG_ENTRY(256, dg::kDense, 2),
    DG_ENTRY(128, dg::kContiguous, 2), DG_ENTRY(160, dg::kContiguous, 2), DG_ENTRY(192, dg::kContiguous, 2),
    DG_ENTRY(224, dg::kContiguous, 2), DG_ENTRY(256, dg::kContiguous, 2),
    DG_BF16_MASKED(64), DG_BF16_MASKED(96), DG_BF16_MASKED(128), DG_BF16_MASKED(160),
    DG_BF16_MASKED(192), DG_BF16_MASKED(224), DG_BF16_MASKED(256),
    DG_LAYOUT(128, 1), DG_LAYOUT(256, 1), DG_LAYOUT(128, 2), DG_LAYOUT(256, 2), DG_LAYOUT(128, 3), DG_LAYOUT(256, 3),
    DG_LAYOUT_PAIR(256, 1), DG_LAYOUT_PAIR(256, 2), DG_LAYOUT_PAIR(256, 3),
    DG_ACC(64, 1), DG_ACC(96, 1), DG_ACC(128, 1), DG_ACC(160, 1), DG_ACC(192, 1), DG_ACC(224, 1), DG_ACC(256, 1),
    DG_ACC(128, 2), DG_ACC(160, 2), DG_ACC(192, 2), DG_ACC(224, 2), DG_ACC(240, 2), DG_ACC(256, 2),
    DG_SMALL_A(64), DG_SMALL_A(96), DG_SMALL_A(128), DG_SMALL_A(160), DG_SMALL_A(192), DG_SMALL_A(224),
    DG_SMALL_A(256),
};
constexpr int kNumKernels = sizeof(kKernels) / sizeof(kKernels[0]);
// 240 (a 16-column tail chunk, double-buffered at nearly 256 columns) is built
// for the dense form on CTA pairs only
constexpr int kBlockNs[] = {64, 96, 128, 160, 192, 224, 240, 256};

// ------------------------------------------------------------------ init ----

// Per-device set-up that allocates no device memory: the driver's tensor-map
// encoder, the architecture check, SM count, kernel attributes, co-resident
// CTA pairs and the address of the status word. Caller holds g_mu.
dg_status setup_device(int dev, DeviceState& st) {
    if (g_encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return DG_ERR_NOT_INITIALIZED;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return DG_ERR_CUDA;
    if (major != 10 || minor != 0) return DG_ERR_UNSUPPORTED;  // built for sm_100a only
    if (cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DG_ERR_CUDA;
    static_assert(kNumKernels <= 80, "DeviceState::max_pairs too small");
    for (int i = 0; i < kNumKernels; ++i) {
        const KernelEntry& e = kKernels[i];
        if (cudaFuncSetAttribute(e.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, e.smem) != cudaSuccess)
            return DG_ERR_CUDA;
        if (e.cg == 2) {
            // how many CTA pairs fit on the device at once (pairs must share a GPC)
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.gridDim = dim3(2 * (st.sms / 2));
            cfg.blockDim = dim3(dg::NUM_THREADS);
            cfg.dynamicSmemBytes = static_cast<size_t>(e.smem);
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, e.fn, &cfg) != cudaSuccess || clusters < 1) return DG_ERR_CUDA;
            st.max_pairs[i] = clusters;
        }
        if (e.cg == 1 && e.kind == dg::kDense && e.layout == 0 && e.dt == dg::kE4M3) {
            // clusters of s CTAs that fit on the device at once (a cluster's CTAs share a GPC)
            for (int s = 2; s <= kMaxClusterSplits; ++s) {
                cudaLaunchConfig_t cfg = {};
                cudaLaunchAttribute attr[1];
                attr[0].id = cudaLaunchAttributeClusterDimension;
                attr[0].val.clusterDim.x = static_cast<unsigned>(s);
                attr[0].val.clusterDim.y = 1;
                attr[0].val.clusterDim.z = 1;
                cfg.gridDim = dim3(static_cast<unsigned>(s * (st.sms / s)));
                cfg.blockDim = dim3(dg::NUM_THREADS);
                cfg.dynamicSmemBytes = static_cast<size_t>(e.smem);
                cfg.attrs = attr;
                cfg.numAttrs = 1;
                int clusters = 0;
                if (cudaOccupancyMaxActiveClusters(&clusters, e.fn, &cfg) != cudaSuccess) {
                    cudaGetLastError();
                    clusters = 0;
                }
                st.max_clusters[i][s] = clusters;
            }
            if (g_log && e.epi == 0)
                std::fprintf(stderr, "[dgb200] BN=%d A-rows=%d: co-resident clusters of 2..8 CTAs: %d %d %d %d %d %d %d\n",
                             e.bn, e.a_rows, st.max_clusters[i][2], st.max_clusters[i][3], st.max_clusters[i][4],
                             st.max_clusters[i][5], st.max_clusters[i][6], st.max_clusters[i][7], st.max_clusters[i][8]);
        }
    }
    void* status = nullptr;
    if (cudaGetSymbolAddress(&status, g_dg_device_status) != cudaSuccess) return DG_ERR_CUDA;
    st.status = static_cast<uint32_t*>(status);
    return DG_OK;
}

// Set up device `dev`, which must be the current device. Allocates nothing.
dg_status init_device(int dev) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (dev < 0 || dev >= kMaxDevices) return DG_ERR_UNSUPPORTED;
    DeviceState& st = g_dev[dev];
    if (st.ready.load(std::memory_order_acquire)) return DG_OK;
    const dg_status s = setup_device(dev, st);
    if (s != DG_OK) return s;
    st.ready.store(true, std::memory_order_release);
    return DG_OK;
}

dg_status noalloc_device(DeviceState** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_NOT_INITIALIZED;
    if (dev < 0 || dev >= kMaxDevices) return DG_ERR_UNSUPPORTED;
    DeviceState& st = g_dev_noalloc[dev];
    if (!st.ready.load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!st.ready.load(std::memory_order_relaxed)) {
            const dg_status s = setup_device(dev, st);
            if (s != DG_OK) return s;
            void* partials = nullptr;
            void* counters = nullptr;
            if (cudaGetSymbolAddress(&partials, g_noalloc_partials) != cudaSuccess ||
                cudaGetSymbolAddress(&counters, g_noalloc_counters) != cudaSuccess)
                return DG_ERR_CUDA;
            st.split_ws = static_cast<float*>(partials);
            st.split_counters = static_cast<uint32_t*>(counters);
            st.ready.store(true, std::memory_order_release);
        }
    }
    *out = &st;
    return DG_OK;
}

dg_status current_device(DeviceState** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_NOT_INITIALIZED;
    if (dev < 0 || dev >= kMaxDevices) return DG_ERR_UNSUPPORTED;
    if (!g_dev[dev].ready.load(std::memory_order_acquire)) {
        dg_status s = init_device(dev);
        if (s != DG_OK) return s;
    }
    *out = &g_dev[dev];
    return DG_OK;
}

// ------------------------------------------------------------ tensor maps --

// K-major operand (k values per row) of 1-byte (E4M3) or 2-byte (BF16)
// elements; the box is one 128-byte row of K by `box_rows` rows.
bool encode_kmajor(CUtensorMap* map, const void* base, int rank, uint64_t k, uint64_t rows, uint64_t mats,
                   uint32_t box_rows, int dt) {
    const uint64_t esz = dt == dg::kBF16 ? 2 : 1;
    cuuint64_t dims[3] = {k, rows, mats};
    cuuint64_t strides[2] = {k * esz, k * esz * rows};  // bytes, dims 1..rank-1
    cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / esz), box_rows, 1};
    cuuint32_t elem[3] = {1, 1, 1};
    const CUtensorMapDataType type = dt == dg::kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    CUresult r = g_encode(map, type, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides, box, elem,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// MN-major E4M3 operand stored [K, mn] (mn contiguous): boxes of 128 bytes of
// mn by 128 K rows with the 128-byte swizzle.
bool encode_mnmajor(CUtensorMap* map, const void* base, uint64_t mn, uint64_t k) {
    cuuint64_t dims[2] = {mn, k};
    cuuint64_t strides[1] = {mn};
    cuuint32_t box[2] = {128, 128};
    cuuint32_t elem[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, elem,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// fp32 output of the dense form (and its C), in boxes of 32 columns x 16 rows
// (128 bytes per row) with the 128-byte swizzle.
bool encode_d_f32(CUtensorMap* map, const void* base, uint64_t n, uint64_t rows) {
    cuuint64_t dims[2] = {n, rows};
    cuuint64_t strides[1] = {4 * n};
    cuuint32_t box[2] = {32, 16};
    cuuint32_t elem[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, elem,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// bf16 output, written by TMA in 32x32 boxes with the 64-byte swizzle.
bool encode_d_bf16(CUtensorMap* map, void* base, int rank, uint64_t n, uint64_t rows, uint64_t mats) {
    cuuint64_t dims[3] = {n, rows, mats};
    cuuint64_t strides[2] = {2 * n, 2 * n * rows};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t elem[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), base, dims, strides,
                          box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------- heuristics --

// Rate at which one SM's TMA loads are fed from L2, in bytes per SM clock
// (about 21 TB/s over 148 SMs at 1.84 GHz, measured with bulk copies of
// L2-resident data into a stage ring while the tensor core runs).
constexpr double kL2BytesPerClk = 77.0;
// Tensor-core clocks lost per tile when the accumulator is single-buffered
// (the MMA warp waits for the epilogue's TMEM reads).
constexpr double kSingleBufferBubble = 600.0;
// Fewest clocks per block-scaled MMA issued from the MMA warp (small N). A
// single CTA streaming a small-M problem (64-row A stages) measured ~150: on
// 64x7168x16384 with 64-wide tiles, 112 CTAs moved 2.97 TB/s, i.e. 8 KB of B
// per ~600 clocks of four MMAs.
constexpr double kMinMmaClocks = 98.0;
constexpr double kMinMmaClocksSmallA = 150.0;
// HBM bytes per SM clock for the whole GPU (~6.5 TB/s at ~1.85 GHz).
constexpr double kHbmBytesPerClk = 3500.0;
// When each B tile is read once (a single m-tile: small M), the weights stream
// from HBM as 128-byte pieces of many rows. Measured on B200: a CTA keeps at
// most `stages` K-blocks in flight and each takes ~2.4 us (4400 clocks) from
// issue to arrival; all CTAs together draw about 2400 bytes per clock.
constexpr double kHbmLatencyClk = 4400.0;
constexpr double kBStreamBytesPerClk = 2400.0;
// One SM streams weights at no more than ~24 bytes per clock (~45 GB/s):
// M = 64 problems measured 40-48 GB/s per streaming SM, so a choice that
// leaves SMs idle cannot make up for them with a faster stream per SM.
constexpr double kBStreamPerSmBytesPerClk = 24.0;
// Split-K through global scratch (fp8_gemm_nt_noalloc): the most ranges per
// tile; the unit that reduces a tile pays about one L2 round trip (~700
// clocks) per 32 columns per two splits, plus a fixed hand-off (fence,
// counter) of ~2000 clocks.
constexpr int kMaxSplits = 16;
constexpr double kL2LatencyClk = 700.0;
constexpr double kSplitFixedClocks = 2000.0;
// Split-K inside a cluster: a fixed hand-off (two cluster-scope barrier
// round trips, ~1500 clocks) plus the pieces each CTA sends to the owners
// through distributed shared memory at about 32 bytes per clock.
constexpr double kClusterSplitFixedClocks = 1500.0;
constexpr double kDsmemBytesPerClk = 32.0;

// Clocks one SM spends per 128-K block of its (rows_a x bn) share of a tile:
// the larger of the tensor core (four K=32 block-scaled MMAs of bn/2 clocks
// each, but no less than ~98 clocks per MMA issued; a pair's MMA covers 128
// rows on each of its two SMs) and the L2 feed of the stage (rows_a rows of A
// and bn/cg rows of B, 128 bytes each).
double kblock_clocks(int bn, int cg, int rows_a, double min_mma = kMinMmaClocks) {
    const double per_mma = bn / 2.0 > min_mma ? bn / 2.0 : min_mma;
    const double tc = 4.0 * per_mma;
    const double l2 = (rows_a + static_cast<double>(bn) / cg) * 128.0 / kL2BytesPerClk;
    return tc > l2 ? tc : l2;
}

// Accumulator slots in TMEM (the kernel's GemmConfig::NUM_ACC).
int num_acc_for(int bn) {
    if (bn % 32 != 0) return 2;  // slots on 256-column boundaries, scale sets in the tails
    return (2 * bn + 2 * (4 + 4 * ((bn + 127) / 128)) <= 512) ? 2 : 1;
}

struct TileChoice {
    const KernelEntry* entry;
    int units;             // concurrent MMA units (CTAs, or CTA pairs); for a cluster split, CTAs
    int splits;            // split-K ranges per output tile (1 = none)
    int split_mode;        // dg::SPLIT_NONE / SPLIT_CLUSTER / SPLIT_SCRATCH
};

// Pick the kernel (N tile, one CTA or a CTA pair) and, for the dense form,
// the split-K factor with the least modelled time: waves of work units over
// the concurrent MMA units x time per unit, but no less than the problem's
// unique bytes at the HBM rate. Split-K is considered only when the output
// tiles alone leave SMs idle; a split unit also pays for writing its fp32
// partial and, on average, for one reduction read of all partials.
// How split-K may run: inside clusters (the library's own calls) or through
// global scratch of the given size (fp8_gemm_nt_noalloc); split_ok false: not
// at all.
struct SplitScratch {
    bool split_ok;
    int mode;             // dg::SPLIT_CLUSTER or dg::SPLIT_SCRATCH
    double bytes;         // SPLIT_SCRATCH: partial bytes available
    long long counters;   // SPLIT_SCRATCH: per-tile counters available
};

TileChoice choose_tile_in(const DeviceState* st, int kind, int rows, int n, int k, long long m128_blocks,
                          long long unique_bytes, int forced_splits, const SplitScratch& scratch, int dt = dg::kE4M3,
                          int layout = 0, int epi = 0) {
    const int kb = k / (dt == dg::kBF16 ? 64 : 128);  // 128-byte rows of K (one pipeline stage each)
    const int kg = (kb + 3) / 4;
    const int forced_bn = g_force_bn.load();
    // no pairs for the masked and psum_m forms
    const int forced_cg = (kind != dg::kMasked && kind != dg::kPsum) ? g_force_cg.load() : 0;
    TileChoice best{nullptr, 0, 1, dg::SPLIT_NONE};
    double best_cost = 1e300;
    const double hbm_floor = static_cast<double>(unique_bytes) / kHbmBytesPerClk;
    for (int i = 0; i < kNumKernels; ++i) {
        const KernelEntry& e = kKernels[i];
        if (e.kind != kind || e.dt != dt || e.layout != layout || e.epi != epi) continue;
        // 64-row A stages serve exactly the dense NT calls with M <= 64 (unless
        // CTA pairs are forced), which use no other kernels
        const bool small_a_call =
            kind == dg::kDense && layout == 0 && epi == 0 && dt == dg::kE4M3 && rows <= 64 && forced_cg != 2;
        if ((e.a_rows < dg::BM) != small_a_call) continue;
        // M <= 64 calls all take 128-column tiles (the split count is still
        // chosen per shape): a small GEMM's first operand loads land several
        // microseconds later when the previous GEMM ran another kernel
        // (cold instruction fetch), which outweighs what a shape-specific
        // width gains alone. Measured on the dense step of 8 problems (four
        // with M = 64): 700 against 730 us per step (median of 21 replays,
        // the one-width step faster in 16 of 21 pairs), although
        // 64x24576x1536 alone takes 13.2 instead of 11.2 us.
        if (small_a_call && forced_bn == 0 && e.bn != 128) continue;
        if (forced_bn != 0 && e.bn != forced_bn) continue;
        if (forced_cg != 0 && e.cg != forced_cg) continue;
        if (forced_cg == 0 && e.cg == 2 && rows < 256) continue;  // a pair needs two row blocks
        // Contiguous pairs only when forced: on the 8-expert 4096x7168 workload
        // they keep the tensor pipe busier (79% vs 74% of cycles) but run at a
        // lower clock under the power cap, and pay ~3% extra work for pairs
        // that span two experts; measured 2% slower than single CTAs.
        if (forced_cg == 0 && e.cg == 2 && kind == dg::kContiguous) continue;
        const int units = e.cg == 1 ? st->sms : st->max_pairs[i];
        if (units < 1) continue;
        const long long mt = (m128_blocks + e.cg - 1) / e.cg;
        const long long nb = (n + e.bn - 1) / e.bn;
        const long long tiles = mt * nb;
        const int rows_a = rows < dg::BM ? rows : dg::BM;
        const double kbc0 = kblock_clocks(e.bn, e.cg, rows_a, e.a_rows < dg::BM ? kMinMmaClocksSmallA : kMinMmaClocks);
        const double bubble = num_acc_for(e.bn) == 1 ? kSingleBufferBubble : 0.0;
        const bool cluster_mode = scratch.mode == dg::SPLIT_CLUSTER;
        const int max_splits = cluster_mode ? kMaxClusterSplits : kMaxSplits;
        for (int splits = 1; splits <= max_splits; ++splits) {
            if (forced_splits != 0 && splits != forced_splits) continue;
            const bool can_split = kind == dg::kDense && e.cg == 1 && e.layout == 0 && scratch.split_ok;
            int su = units;  // concurrent work units of this split count
            if (splits > 1) {
                if (!can_split || splits > kg) break;
                if (cluster_mode) {
                    // every CTA owns at least one 8-column piece; the received
                    // pieces fit in the operand ring
                    if (splits > e.bn / 8) break;
                    if (dg::cluster_split_bytes(e.bn, splits) > e.stages * e.stage_bytes) continue;
                    su = st->max_clusters[i][splits] * splits;
                    if (su < splits) continue;
                } else {
                    if (tiles > scratch.counters) break;
                    if (static_cast<double>(tiles) * splits * dg::BM * e.bn * sizeof(float) > scratch.bytes) break;
                }
                if (forced_splits == 0 && tiles >= units) break;  // the tiles alone fill the GPU
            }
            const int gps = (kg + splits - 1) / splits;  // K groups of the longest range
            const long long work = tiles * splits;
            const long long waves = (work + su - 1) / su;
            const int kb_unit = gps * 4 < kb ? gps * 4 : kb;
            double kbc = kbc0;
            if (mt == 1) {  // B streamed once from HBM
                const double active = static_cast<double>(work < su ? work : su);
                const double lat = kHbmLatencyClk / e.stages;
                const double bw = static_cast<double>(e.bn / e.cg) * 128.0 * active / kBStreamBytesPerClk;
                const double per_sm = static_cast<double>(e.bn / e.cg) * 128.0 / kBStreamPerSmBytesPerClk;
                if (lat > kbc) kbc = lat;
                if (bw > kbc) kbc = bw;
                if (per_sm > kbc) kbc = per_sm;
            }
            double unit = kb_unit * kbc + bubble;
            if (splits > 1) {
                if (cluster_mode)
                    unit += kClusterSplitFixedClocks +
                            static_cast<double>(rows_a) * e.bn * 4.0 * (splits - 1) / splits / kDsmemBytesPerClk;
                else
                    unit += (e.bn / 32.0) * ((splits + 1) / 2) * kL2LatencyClk + kSplitFixedClocks;
            }
            double cost = static_cast<double>(waves) * unit;
            if (cost < hbm_floor) cost = hbm_floor;
            const bool better =
                cost < best_cost * 0.999 ||
                (cost <= best_cost * 1.001 && best.entry &&
                 (splits < best.splits ||
                  (splits == best.splits && (e.cg > best.entry->cg || (e.cg == best.entry->cg && e.bn > best.entry->bn)))));
            if (best.entry == nullptr || better) {
                best_cost = cost;
                best = TileChoice{&e, su, splits, splits > 1 ? scratch.mode : dg::SPLIT_NONE};
            }
        }
    }
    return best;
}

// The library's own choice: split-K inside clusters, and the split count
// forced by dgb200_set_splits (dense form).
TileChoice choose_tile(const DeviceState* st, int kind, int rows, int n, int k, long long m128_blocks,
                       long long unique_bytes, int dt = dg::kE4M3, int layout = 0, int epi = 0) {
    const int forced_splits = kind == dg::kDense ? g_force_splits.load() : 1;
    const SplitScratch scratch{true, dg::SPLIT_CLUSTER, 0.0, 0};
    return choose_tile_in(st, kind, rows, n, k, m128_blocks, unique_bytes, forced_splits, scratch, dt, layout, epi);
}

// Launch configuration of the elementwise pack kernels (programmatic
// serialization as for the GEMMs); `attr` must outlive the launch call.
cudaLaunchConfig_t small_launch(unsigned blocks, int threads, void* stream, cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.stream = static_cast<cudaStream_t>(stream);
    if (g_pdl) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cfg;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

dg_status check_common(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, const void* d, int N,
                       int K) {
    if (!a || !sfa || !b || !sfb || !d) return DG_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0) return DG_ERR_INVALID_ARG;
    if (K % 128 != 0 || N % 8 != 0) return DG_ERR_INVALID_ARG;
    if (K > (1 << 20)) return DG_ERR_UNSUPPORTED;
    if (!aligned(a, 16) || !aligned(b, 16) || !aligned(d, 16) || !aligned(sfa, 4) || !aligned(sfb, 4))
        return DG_ERR_ALIGNMENT;
    return DG_OK;
}

// Launch one GEMM with a given tile choice; split-K partials and counters
// come from `ws` / `counters` (used only when the choice splits through
// global scratch).
dg_status launch_gemm_with(const TileChoice& choice, float* ws, uint32_t* counters, int kind, GemmParams& p,
                           long long max_tiles_per_nblock, void* stream, const DeviceState* st, const void* a,
                           const void* b, int a_rank, int b_rank, uint64_t a_rows, uint64_t a_mats, uint64_t b_rows,
                           uint64_t b_mats) {
    const KernelEntry* e = choice.entry;
    if (e == nullptr) return DG_ERR_UNSUPPORTED;
    const int bn = e->bn;
    const int cg = e->cg;
    p.status = st->status;
    p.kb = p.k / (e->dt == dg::kBF16 ? 64 : 128);  // 128-byte rows of K per operand row
    p.kp = (p.kb + 3) / 4;
    p.nb_sf = p.sfb_per_row ? p.n : (p.n + 127) / 128;
    // 16-byte reads of the scale rows need every row to start on a 16-byte boundary
    p.sf_vec4 = ((p.sfb_per_row || kind == dg::kDense) && e->dt == dg::kE4M3 && g_sf_vec4 && p.kp % 4 == 0 &&
                 aligned(p.sfa, 16) && (!p.sfb_per_row || aligned(p.sfb, 16)))
                    ? 1
                    : 0;
    p.num_n_blocks = (p.n + bn - 1) / bn;
    if (cg == 2) p.num_m_blocks = (p.rows + 2 * dg::BM - 1) / (2 * dg::BM);
    // bands of 2048 rows (measured on 4096x7168x16384: taller bands, which
    // would read each weight tile from DRAM only once, thrash L2 with A and
    // read more, 592 MB against 473 MB)
    p.raster_group = 16 / cg;
    p.raster_shift = cg == 2 ? 3 : 4;
    p.inv_band_tiles = 1.0f / static_cast<float>(p.raster_group * p.num_n_blocks);
    p.wait_limit_ns = g_wait_limit_ns.load();
    p.test_mode = g_test_mode.load();
    p.splits = choice.splits;
    p.split_mode = choice.splits > 1 ? choice.split_mode : dg::SPLIT_NONE;
    const bool scratch_split = p.split_mode == dg::SPLIT_SCRATCH;
    if (scratch_split && (ws == nullptr || counters == nullptr)) return DG_ERR_UNSUPPORTED;
    p.ws = scratch_split ? ws : nullptr;
    p.counters = scratch_split ? counters : nullptr;
    p.k_rotate = choice.splits > 1 ? 0 : g_k_rotate;  // a split walks its own range in order
    if (p.k_rotate) p.sf_vec4 = 0;                     // quads are walked in K order
    if (e->layout & 1) {
        if (!encode_mnmajor(&p.tma_a, a, a_rows, static_cast<uint64_t>(p.k))) return DG_ERR_INVALID_ARG;
    } else if (!encode_kmajor(&p.tma_a, a, a_rank, static_cast<uint64_t>(p.k), a_rows, a_mats,
                              static_cast<uint32_t>(e->a_rows), e->dt)) {
        return DG_ERR_INVALID_ARG;
    }
    if (e->layout & 2) {
        if (!encode_mnmajor(&p.tma_b, b, b_rows, static_cast<uint64_t>(p.k))) return DG_ERR_INVALID_ARG;
    } else if (!encode_kmajor(&p.tma_b, b, b_rank, static_cast<uint64_t>(p.k), b_rows, b_mats,
                              static_cast<uint32_t>(bn / cg), e->dt)) {
        return DG_ERR_INVALID_ARG;
    }
    if (!encode_d_bf16(&p.tma_d, p.d, a_rank, static_cast<uint64_t>(p.n), a_rows, a_mats)) return DG_ERR_INVALID_ARG;
    if (kind == dg::kDense && p.out_f32 &&
        !encode_d_f32(&p.tma_d, p.d32, static_cast<uint64_t>(p.n), static_cast<uint64_t>(p.rows)))
        return DG_ERR_INVALID_ARG;
    if (kind == dg::kDense && p.c != nullptr) {
        const bool ok = p.out_f32 ? encode_d_f32(&p.tma_c, p.c, static_cast<uint64_t>(p.n), static_cast<uint64_t>(p.rows))
                                  : encode_d_bf16(&p.tma_c, const_cast<void*>(p.c), 2, static_cast<uint64_t>(p.n),
                                                  static_cast<uint64_t>(p.rows), 1);
        if (!ok) return DG_ERR_INVALID_ARG;
    }
    // contiguous pairs walk two passes (see next_tile in gemm_kernel.cuh)
    const long long tiles = (cg == 1 ? max_tiles_per_nblock : p.num_m_blocks) * static_cast<long long>(p.num_n_blocks) *
                            choice.splits * (cg == 2 && kind == dg::kContiguous ? 2 : 1);
    if (tiles <= 0) return DG_OK;
    // a cluster split runs every work unit on a CTA of its own (one tile per
    // cluster: the reduction uses the operand ring, which is then idle)
    const bool cluster_split = p.split_mode == dg::SPLIT_CLUSTER;
    if (cluster_split && (kind != dg::kDense || cg != 1 || tiles > (1LL << 30))) return DG_ERR_UNSUPPORTED;
    const int units = cluster_split ? static_cast<int>(tiles)
                                    : static_cast<int>(tiles < choice.units ? tiles : choice.units);
    void* args[] = {&p};
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    unsigned nattr = 0;
    if (cg == 2 || cluster_split) {
        attr[nattr].id = cudaLaunchAttributeClusterDimension;
        attr[nattr].val.clusterDim.x = cg == 2 ? 2u : static_cast<unsigned>(choice.splits);
        attr[nattr].val.clusterDim.y = 1;
        attr[nattr].val.clusterDim.z = 1;
        ++nattr;
    }
    if (g_pdl) {
        attr[nattr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[nattr].val.programmaticStreamSerializationAllowed = 1;
        ++nattr;
    }
    cfg.gridDim = dim3(static_cast<unsigned>(units * cg));
    cfg.blockDim = dim3(dg::NUM_THREADS);
    cfg.dynamicSmemBytes = static_cast<size_t>(e->smem);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cfg.attrs = attr;
    cfg.numAttrs = nattr;
    if (g_log)
        std::fprintf(stderr,
                     "[dgb200] form=%d rows=%d N=%d K=%d groups=%d: BN=%d CTA-group=%d splits=%d (mode %d) grid=%d "
                     "(units %d) smem=%d stages=%d A-rows=%d\n",
                     kind, p.rows, p.n, p.k, p.groups, bn, cg, choice.splits, p.split_mode, units * cg, choice.units,
                     e->smem, e->stages, e->a_rows);
    cudaError_t err = cudaLaunchKernelExC(&cfg, e->fn, args);
    return err == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

dg_status launch_gemm(int kind, GemmParams& p, long long m_blocks_for_heuristic, long long max_tiles_per_nblock,
                      long long unique_bytes, void* stream, DeviceState* st, const void* a, const void* b, int a_rank,
                      int b_rank, uint64_t a_rows, uint64_t a_mats, uint64_t b_rows, uint64_t b_mats,
                      int dt = dg::kE4M3, int layout = 0, int epi = 0) {
    const TileChoice choice =
        choose_tile(st, kind, p.rows, p.n, p.k, m_blocks_for_heuristic, unique_bytes, dt, layout, epi);
    return launch_gemm_with(choice, nullptr, nullptr, kind, p, max_tiles_per_nblock, stream, st, a, b, a_rank, b_rank,
                            a_rows, a_mats, b_rows, b_mats);
}

// Scale rows of B: one per 128x128 block (sfb_gran_n = 128) or one per row of B
// (sfb_gran_n = 1).
dg_status sfb_granularity(int sfb_gran_n, int* per_row) {
    if (sfb_gran_n != 128 && sfb_gran_n != 1) return DG_ERR_INVALID_ARG;
    *per_row = sfb_gran_n == 1;
    return DG_OK;
}

// Dense NT GEMM, D = C + A.B^T. Without C and with a bf16 D it runs the plain
// epilogue; otherwise the instantiations that add C and/or store fp32.
dg_status dense_nt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, int sfb_per_row, const void* c,
                   void* d, int M, int N, int K, int out_f32, void* stream) {
    dg_status s = check_common(a, sfa, b, sfb, d, N, K);
    if (s != DG_OK) return s;
    if (M <= 0 || (out_f32 != 0 && out_f32 != 1)) return DG_ERR_INVALID_ARG;
    if (c != nullptr && !aligned(c, 16)) return DG_ERR_ALIGNMENT;
    DeviceState* st = nullptr;
    if ((s = current_device(&st)) != DG_OK) return s;
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.sfa = sfa;
    p.sfb = sfb;
    p.sfb_per_row = sfb_per_row;
    p.d = static_cast<__nv_bfloat16*>(d);  // bf16 output (the D tensor map covers it either way)
    p.d32 = out_f32 ? static_cast<float*>(d) : nullptr;
    p.out_f32 = out_f32;
    p.c = c;
    p.meta = nullptr;
    p.rows = M;
    p.n = N;
    p.k = K;
    p.groups = 1;
    p.num_m_blocks = (M + dg::BM - 1) / dg::BM;
    const long long esz = out_f32 ? 4 : 2;
    const long long bytes = (static_cast<long long>(M) + N) * K + esz * M * N * (c != nullptr ? 2 : 1);
    const int epi = (c != nullptr || out_f32) ? 1 : 0;
    return launch_gemm(dg::kDense, p, p.num_m_blocks, p.num_m_blocks, bytes, stream, st, a, b, 2, 2,
                       static_cast<uint64_t>(M), 1, static_cast<uint64_t>(N), 1, dg::kE4M3, 0, epi);
}

dg_status contiguous_nt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, int sfb_per_row,
                        void* d, const int32_t* m_indices, int M_total, int N, int K, int G, void* stream) {
    dg_status s = check_common(a, sfa, b, sfb, d, N, K);
    if (s != DG_OK) return s;
    if (M_total <= 0 || G <= 0 || m_indices == nullptr) return DG_ERR_INVALID_ARG;
    if (!aligned(m_indices, 4)) return DG_ERR_ALIGNMENT;
    DeviceState* st = nullptr;
    if ((s = current_device(&st)) != DG_OK) return s;
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.sfa = sfa;
    p.sfb = sfb;
    p.sfb_per_row = sfb_per_row;
    p.d = static_cast<__nv_bfloat16*>(d);
    p.meta = m_indices;
    p.rows = M_total;
    p.n = N;
    p.k = K;
    p.groups = G;
    p.num_m_blocks = (M_total + dg::BM - 1) / dg::BM;
    const long long bytes = static_cast<long long>(M_total) * K + static_cast<long long>(G) * N * K +
                            2LL * M_total * N;
    return launch_gemm(dg::kContiguous, p, p.num_m_blocks, p.num_m_blocks, bytes, stream, st, a, b, 2, 3,
                       static_cast<uint64_t>(M_total), 1, static_cast<uint64_t>(N), static_cast<uint64_t>(G));
}

dg_status masked_nt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, int sfb_per_row, void* d,
                    const int32_t* masked_m, int G, int max_m, int N, int K, void* stream) {
    dg_status s = check_common(a, sfa, b, sfb, d, N, K);
    if (s != DG_OK) return s;
    if (G <= 0 || max_m <= 0 || masked_m == nullptr) return DG_ERR_INVALID_ARG;
    if (G > dg::MAX_MASKED_GROUPS) return DG_ERR_UNSUPPORTED;
    if (!aligned(masked_m, 4)) return DG_ERR_ALIGNMENT;
    DeviceState* st = nullptr;
    if ((s = current_device(&st)) != DG_OK) return s;
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.sfa = sfa;
    p.sfb = sfb;
    p.sfb_per_row = sfb_per_row;
    p.d = static_cast<__nv_bfloat16*>(d);
    p.meta = masked_m;
    p.rows = max_m;
    p.n = N;
    p.k = K;
    p.groups = G;
    p.num_m_blocks = (max_m + dg::BM - 1) / dg::BM;
    const long long mb_total = static_cast<long long>(G) * p.num_m_blocks;
    const long long bytes = static_cast<long long>(G) * N * K;  // the weights; the valid rows are unknown here
    return launch_gemm(dg::kMasked, p, mb_total, mb_total, bytes, stream, st, a, b, 3, 3, static_cast<uint64_t>(max_m),
                       static_cast<uint64_t>(G), static_cast<uint64_t>(N), static_cast<uint64_t>(G));
}

// psum_m form: A [M_total, K] with the groups' rows end to end, group g
// owning rows [psum_m[g-1], psum_m[g]); D [M_total, N]; B [G, N, K].
dg_status psum_nt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d,
                  const int32_t* psum_m, int M_total, int N, int K, int G, void* stream) {
    dg_status s = check_common(a, sfa, b, sfb, d, N, K);
    if (s != DG_OK) return s;
    if (M_total <= 0 || G <= 0 || psum_m == nullptr) return DG_ERR_INVALID_ARG;
    if (G > dg::MAX_MASKED_GROUPS) return DG_ERR_UNSUPPORTED;
    if (!aligned(psum_m, 4)) return DG_ERR_ALIGNMENT;
    DeviceState* st = nullptr;
    if ((s = current_device(&st)) != DG_OK) return s;
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.sfa = sfa;
    p.sfb = sfb;
    p.d = static_cast<__nv_bfloat16*>(d);
    p.meta = psum_m;
    p.rows = M_total;
    p.n = N;
    p.k = K;
    p.groups = G;
    p.num_m_blocks = (M_total + dg::BM - 1) / dg::BM;
    // a group boundary inside a 128-row block adds at most one block per group
    const long long mb_total = static_cast<long long>(p.num_m_blocks) + G;
    const long long bytes = static_cast<long long>(M_total) * K + static_cast<long long>(G) * N * K +
                            2LL * M_total * N;
    return launch_gemm(dg::kPsum, p, mb_total, mb_total, bytes, stream, st, a, b, 2, 3,
                       static_cast<uint64_t>(M_total), 1, static_cast<uint64_t>(N), static_cast<uint64_t>(G));
}

}  // namespace

extern "C" {

const char* dgb200_status_string(dg_status s) {
    switch (s) {
        case DG_OK: return "DG_OK";
        case DG_ERR_INVALID_ARG: return "DG_ERR_INVALID_ARG";
        case DG_ERR_ALIGNMENT: return "DG_ERR_ALIGNMENT";
        case DG_ERR_UNSUPPORTED: return "DG_ERR_UNSUPPORTED";
        case DG_ERR_NOT_INITIALIZED: return "DG_ERR_NOT_INITIALIZED";
        case DG_ERR_CUDA: return "DG_ERR_CUDA";
        case DG_ERR_SCRATCH_TOO_SMALL: return "DG_ERR_SCRATCH_TOO_SMALL";
    }
    return "DG_ERR_UNKNOWN";
}

dg_status dgb200_init(int device) {
    int count = 0;
    if (cudaGetDeviceCount(&count) != cudaSuccess) {
        cudaGetLastError();
        return DG_ERR_NOT_INITIALIZED;
    }
    if (device < 0 || device >= count) return DG_ERR_INVALID_ARG;
    if (device >= kMaxDevices) return DG_ERR_UNSUPPORTED;
    if (g_dev[device].ready.load(std::memory_order_acquire)) return DG_OK;
    // kernel attributes apply to the current device: make `device` current for
    // the set-up and restore the caller's device afterwards
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) return DG_ERR_NOT_INITIALIZED;
    if (prev != device && cudaSetDevice(device) != cudaSuccess) return DG_ERR_CUDA;
    const dg_status s = init_device(device);
    if (prev != device && cudaSetDevice(prev) != cudaSuccess) return DG_ERR_CUDA;
    return s;
}

// Address of the status word on the current device without setting up the
// kernels (the word is a static variable of the library's module).
dg_status status_word(uint32_t** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_NOT_INITIALIZED;
    if (dev < 0 || dev >= kMaxDevices) return DG_ERR_UNSUPPORTED;
    void* status = nullptr;
    if (cudaGetSymbolAddress(&status, g_dg_device_status) != cudaSuccess) return DG_ERR_CUDA;
    *out = static_cast<uint32_t*>(status);
    return DG_OK;
}

dg_status dgb200_device_error(uint32_t* bits, int clear) {
    if (bits == nullptr) return DG_ERR_INVALID_ARG;
    uint32_t* word = nullptr;
    const dg_status s = status_word(&word);
    if (s != DG_OK) return s;
    if (cudaDeviceSynchronize() != cudaSuccess) return DG_ERR_CUDA;
    if (cudaMemcpy(bits, word, sizeof(uint32_t), cudaMemcpyDeviceToHost) != cudaSuccess) return DG_ERR_CUDA;
    if (clear && cudaMemset(word, 0, sizeof(uint32_t)) != cudaSuccess) return DG_ERR_CUDA;
    if (clear && cudaDeviceSynchronize() != cudaSuccess) return DG_ERR_CUDA;
    return DG_OK;
}

dg_status dgb200_last_device_error(int* code) {
    if (code == nullptr) return DG_ERR_INVALID_ARG;
    uint32_t bits = 0;
    const dg_status s = dgb200_device_error(&bits, 1);
    if (s != DG_OK) return s;
    *code = static_cast<int>(bits);
    return DG_OK;
}

int dgb200_block_n_supported(int block_n) {
    for (int bn : kBlockNs)
        if (bn == block_n) return 1;
    return 0;
}

dg_status dgb200_set_block_n(int block_n) {
    if (block_n != 0 && !dgb200_block_n_supported(block_n)) return DG_ERR_UNSUPPORTED;
    g_force_bn.store(block_n);
    return DG_OK;
}

dg_status dgb200_set_cta_group(int cta_group) {
    if (cta_group < 0 || cta_group > 2) return DG_ERR_UNSUPPORTED;
    g_force_cg.store(cta_group);
    return DG_OK;
}

dg_status dgb200_set_splits(int splits) {
    if (splits < 0 || splits > kMaxClusterSplits) return DG_ERR_UNSUPPORTED;
    g_force_splits.store(splits);
    return DG_OK;
}

dg_status dgb200_set_test_hooks(int mode, int wait_limit_ms) {
    if (mode < 0 || mode > 1 || wait_limit_ms < 0) return DG_ERR_INVALID_ARG;
    g_test_mode.store(mode);
    g_wait_limit_ns.store(wait_limit_ms == 0 ? dg::DEFAULT_WAIT_LIMIT_NS
                                             : static_cast<uint64_t>(wait_limit_ms) * 1000000ull);
    return DG_OK;
}

dg_status fp8_gemm_nt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d, int M, int N,
                      int K, void* stream) {
    return dense_nt(a, sfa, b, sfb, 0, nullptr, d, M, N, K, 0, stream);
}

// Dense GEMM in the TN/NN/TT layouts (layout bit 0: A stored [K, M]; bit 1: B
// stored [K, N]).
dg_status fp8_gemm_layout(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d, int M, int N,
                          int K, int layout, void* stream) {
    dg_status s = check_common(a, sfa, b, sfb, d, N, K);
    if (s != DG_OK) return s;
    if (M <= 0) return DG_ERR_INVALID_ARG;
    if (((layout & 1) && M % 16 != 0) || ((layout & 2) && N % 16 != 0)) return DG_ERR_INVALID_ARG;
    DeviceState* st = nullptr;
    if ((s = current_device(&st)) != DG_OK) return s;
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.sfa = sfa;
    p.sfb = sfb;
    p.d = static_cast<__nv_bfloat16*>(d);
    p.rows = M;
    p.n = N;
    p.k = K;
    p.groups = 1;
    p.num_m_blocks = (M + dg::BM - 1) / dg::BM;
    const long long bytes = (static_cast<long long>(M) + N) * K + 2LL * M * N;
    return launch_gemm(dg::kDense, p, p.num_m_blocks, p.num_m_blocks, bytes, stream, st, a, b, 2, 2,
                       static_cast<uint64_t>(M), 1, static_cast<uint64_t>(N), 1, dg::kE4M3, layout);
}

dg_status fp8_gemm_nn(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d, int M, int N,
                      int K, void* stream) {
    return fp8_gemm_layout(a, sfa, b, sfb, d, M, N, K, 2, stream);
}

dg_status fp8_gemm_tn(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d, int M, int N,
                      int K, void* stream) {
    return fp8_gemm_layout(a, sfa, b, sfb, d, M, N, K, 3, stream);
}

dg_status fp8_gemm_tt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d, int M, int N,
                      int K, void* stream) {
    return fp8_gemm_layout(a, sfa, b, sfb, d, M, N, K, 1, stream);
}

dg_status fp8_gemm_nt_acc(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, const void* c, void* d,
                          int M, int N, int K, int out_f32, void* stream) {
    return dense_nt(a, sfa, b, sfb, 0, c, d, M, N, K, out_f32, stream);
}

dg_status fp8_gemm_nt_sfb_gran(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, int sfb_gran_n,
                               const void* c, void* d, int M, int N, int K, int out_f32, void* stream) {
    int per_row = 0;
    const dg_status s = sfb_granularity(sfb_gran_n, &per_row);
    if (s != DG_OK) return s;
    return dense_nt(a, sfa, b, sfb, per_row, c, d, M, N, K, out_f32, stream);
}

dg_status fp8_gemm_nt_noalloc(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d, int M,
                              int N, int K, int splits, void* stream) {
    dg_status s = check_common(a, sfa, b, sfb, d, N, K);
    if (s != DG_OK) return s;
    if (M <= 0) return DG_ERR_INVALID_ARG;
    if (splits < 0 || splits > kMaxSplits) return DG_ERR_UNSUPPORTED;
    DeviceState* st = nullptr;
    if ((s = noalloc_device(&st)) != DG_OK) return s;
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.sfa = sfa;
    p.sfb = sfb;
    p.d = static_cast<__nv_bfloat16*>(d);
    p.meta = nullptr;
    p.rows = M;
    p.n = N;
    p.k = K;
    p.groups = 1;
    p.num_m_blocks = (M + dg::BM - 1) / dg::BM;
    const long long bytes = (static_cast<long long>(M) + N) * K + 2LL * M * N;
    const double static_bytes = static_cast<double>(kStaticPartialFloats) * sizeof(float);
    // the model's choice among the tile widths whose partials fit the static
    // scratch (splits = 0: any split count; else exactly `splits`)
    const SplitScratch scratch{true, dg::SPLIT_SCRATCH, static_bytes, kStaticCounters};
    const TileChoice choice = choose_tile_in(st, dg::kDense, M, N, K, p.num_m_blocks, bytes, splits, scratch);
    if (choice.entry == nullptr) {
        // refused: say whether scratch without limits would have allowed it
        const SplitScratch unlimited{true, dg::SPLIT_SCRATCH, 1e300, 1LL << 40};
        const TileChoice any = choose_tile_in(st, dg::kDense, M, N, K, p.num_m_blocks, bytes, splits, unlimited);
        return any.entry != nullptr ? DG_ERR_SCRATCH_TOO_SMALL : DG_ERR_UNSUPPORTED;
    }
    if (choice.splits > 1) {
        // the counters must start at zero (a launch that gave up may have left some part-way)
        const long long tiles = p.num_m_blocks * ((N + choice.entry->bn - 1) / choice.entry->bn);
        if (cudaMemsetAsync(st->split_counters, 0, static_cast<size_t>(tiles) * sizeof(uint32_t),
                            static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return DG_ERR_CUDA;
    }
    return launch_gemm_with(choice, st->split_ws, st->split_counters, dg::kDense, p, p.num_m_blocks, stream, st, a, b,
                            2, 2, static_cast<uint64_t>(M), 1, static_cast<uint64_t>(N), 1);
}

dg_status m_grouped_fp8_gemm_nt_contiguous(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                           void* d, const int32_t* m_indices, int M_total, int N, int K, int G,
                                           void* stream) {
    return contiguous_nt(a, sfa, b, sfb, 0, d, m_indices, M_total, N, K, G, stream);
}

dg_status m_grouped_fp8_gemm_nt_contiguous_sfb_gran(const void* a, const int32_t* sfa, const void* b,
                                                    const int32_t* sfb, int sfb_gran_n, void* d,
                                                    const int32_t* m_indices, int M_total, int N, int K, int G,
                                                    void* stream) {
    int per_row = 0;
    const dg_status s = sfb_granularity(sfb_gran_n, &per_row);
    if (s != DG_OK) return s;
    return contiguous_nt(a, sfa, b, sfb, per_row, d, m_indices, M_total, N, K, G, stream);
}

dg_status m_grouped_fp8_gemm_nt_masked(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d,
                                       const int32_t* masked_m, int G, int max_m, int N, int K, void* stream) {
    return masked_nt(a, sfa, b, sfb, 0, d, masked_m, G, max_m, N, K, stream);
}

dg_status m_grouped_fp8_gemm_nt_masked_sfb_gran(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb,
                                                int sfb_gran_n, void* d, const int32_t* masked_m, int G, int max_m,
                                                int N, int K, void* stream) {
    int per_row = 0;
    const dg_status s = sfb_granularity(sfb_gran_n, &per_row);
    if (s != DG_OK) return s;
    return masked_nt(a, sfa, b, sfb, per_row, d, masked_m, G, max_m, N, K, stream);
}

dg_status m_grouped_fp8_gemm_nt_psum(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d,
                                     const int32_t* psum_m, int M_total, int N, int K, int G, void* stream) {
    return psum_nt(a, sfa, b, sfb, d, psum_m, M_total, N, K, G, stream);
}

dg_status m_grouped_bf16_gemm_nt_masked(const void* a, const void* b, void* d, const int32_t* masked_m, int G,
                                        int max_m, int N, int K, void* stream) {
    if (!a || !b || !d || !masked_m) return DG_ERR_INVALID_ARG;
    if (G <= 0 || max_m <= 0 || N <= 0 || K <= 0) return DG_ERR_INVALID_ARG;
    if (K % 64 != 0 || N % 8 != 0) return DG_ERR_INVALID_ARG;
    if (G > dg::MAX_MASKED_GROUPS) return DG_ERR_UNSUPPORTED;
    if (!aligned(a, 16) || !aligned(b, 16) || !aligned(d, 16) || !aligned(masked_m, 4)) return DG_ERR_ALIGNMENT;
    DeviceState* st = nullptr;
    dg_status s = current_device(&st);
    if (s != DG_OK) return s;
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.d = static_cast<__nv_bfloat16*>(d);
    p.meta = masked_m;
    p.rows = max_m;
    p.n = N;
    p.k = K;
    p.groups = G;
    p.num_m_blocks = (max_m + dg::BM - 1) / dg::BM;
    const long long mb_total = static_cast<long long>(G) * p.num_m_blocks;
    const long long bytes = 2LL * G * N * K;  // the weights; the valid rows are unknown here
    return launch_gemm(dg::kMasked, p, mb_total, mb_total, bytes, stream, st, a, b, 3, 3, static_cast<uint64_t>(max_m),
                       static_cast<uint64_t>(G), static_cast<uint64_t>(N), static_cast<uint64_t>(G), dg::kBF16);
}

dg_status pack_ue8m0(const float* sf, int32_t* packed, int64_t rows, int cols, void* stream) {
    if (!sf || !packed || rows <= 0 || cols <= 0) return DG_ERR_INVALID_ARG;
    if (!aligned(sf, 4) || !aligned(packed, 4)) return DG_ERR_ALIGNMENT;
    DeviceState* st = nullptr;
    dg_status s = current_device(&st);
    if (s != DG_OK) return s;
    const int kp = (cols + 3) / 4;
    const int64_t words = rows * kp;
    const int threads = 256;
    int64_t blocks = (words + threads - 1) / threads;
    const int64_t cap = static_cast<int64_t>(st->sms) * 8;
    if (blocks > cap) blocks = cap;
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = small_launch(static_cast<unsigned>(blocks), threads, stream, attr);
    cudaError_t err;
    if (cols % 4 == 0 && aligned(sf, 16)) {
        err = cudaLaunchKernelEx(&cfg, dg::pack_ue8m0_vec4_kernel, reinterpret_cast<const float4*>(sf),
                                 reinterpret_cast<uint32_t*>(packed), words);
    } else {
        err = cudaLaunchKernelEx(&cfg, dg::pack_ue8m0_rows_kernel, sf, reinterpret_cast<uint32_t*>(packed), rows, cols,
                                 kp);
    }
    return err == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

dg_status quantize_fp8_1x128(const void* x, int x_f32, void* q, int32_t* sf_packed, float* sf_f32, int64_t rows, int K,
                             void* stream) {
    if (!x || !q || !sf_packed || rows <= 0 || K <= 0 || (x_f32 != 0 && x_f32 != 1)) return DG_ERR_INVALID_ARG;
    if (K % 128 != 0) return DG_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(sf_packed, 4) || (sf_f32 && !aligned(sf_f32, 4)))
        return DG_ERR_ALIGNMENT;
    DeviceState* st = nullptr;
    dg_status s = current_device(&st);
    if (s != DG_OK) return s;
    const int kb = K / 128;
    const int kp = (kb + 3) / 4;
    const int threads = dg::QUANT_THREADS;
    const int64_t warps_needed = (rows * kb + dg::QUANT_UNROLL - 1) / dg::QUANT_UNROLL;
    int64_t blocks = (warps_needed + threads / 32 - 1) / (threads / 32);
    const int64_t cap = static_cast<int64_t>(st->sms) * dg::QUANT_BLOCKS_PER_SM;
    if (blocks > cap) blocks = cap;
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = small_launch(static_cast<unsigned>(blocks), threads, stream, attr);
    uint32_t* qw = static_cast<uint32_t*>(q);
    uint8_t* sb = reinterpret_cast<uint8_t*>(sf_packed);
    const cudaError_t err =
        x_f32 ? cudaLaunchKernelEx(&cfg, dg::quantize_fp8_1x128_kernel<true>, x, qw, sb, sf_f32, rows, kb, kp)
              : cudaLaunchKernelEx(&cfg, dg::quantize_fp8_1x128_kernel<false>, x, qw, sb, sf_f32, rows, kb, kp);
    return err == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

dg_status pack_ue8m0_validate(const float* sf, int64_t rows, int cols, int32_t* bad_count, void* stream) {
    if (!sf || !bad_count || rows <= 0 || cols <= 0) return DG_ERR_INVALID_ARG;
    if (!aligned(sf, 4) || !aligned(bad_count, 4)) return DG_ERR_ALIGNMENT;
    DeviceState* st = nullptr;
    dg_status s = current_device(&st);
    if (s != DG_OK) return s;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(bad_count, 0, sizeof(int32_t), cs) != cudaSuccess) return DG_ERR_CUDA;
    const int64_t n = rows * cols;
    const int threads = 256;
    int64_t blocks = (n + threads - 1) / threads;
    const int64_t cap = static_cast<int64_t>(st->sms) * 8;
    if (blocks > cap) blocks = cap;
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = small_launch(static_cast<unsigned>(blocks), threads, stream, attr);
    const cudaError_t err = cudaLaunchKernelEx(&cfg, dg::pack_ue8m0_validate_kernel, sf, n, bad_count);
    return err == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

}  // extern "C"
