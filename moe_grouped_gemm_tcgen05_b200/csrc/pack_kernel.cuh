// Capture-safe UE8M0 pack and its optional validator.
//
// "[GH-ISSUE #414] pack_ue8m0_to_int is not CUDA Graph capture safe", Expected
// behavior: the pack is the biased-exponent byte of each fp32 scale
// ((bits >> 23), low 8 bits), four consecutive bytes per int32, little-endian;
// the value checks (sign clear, mantissa zero) belong on a separate eager path.
// Neither kernel reads a device value back to the host.
#pragma once

#include <cstdint>
#include <type_traits>

#include "ptx.cuh"

namespace dg {

__device__ __forceinline__ uint32_t ue8m0_byte(float x) {
    return (__float_as_uint(x) >> 23) & 0xFFu;
}

// cols % 4 == 0 and 16-byte aligned input: word i packs floats 4i..4i+3, so the
// whole tensor is one flat stream of float4 -> int32.
__global__ void pack_ue8m0_vec4_kernel(const float4* __restrict__ sf, uint32_t* __restrict__ out, int64_t words) {
    griddep_launch_dependents();
    griddep_wait();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < words; i += stride) {
        const float4 v = __ldg(sf + i);
        out[i] = ue8m0_byte(v.x) | (ue8m0_byte(v.y) << 8) | (ue8m0_byte(v.z) << 16) | (ue8m0_byte(v.w) << 24);
    }
}

// General layout: rows x cols floats -> rows x kp words, zero bytes past cols.
__global__ void pack_ue8m0_rows_kernel(const float* __restrict__ sf, uint32_t* __restrict__ out, int64_t rows,
                                       int cols, int kp) {
    griddep_launch_dependents();
    griddep_wait();
    const int64_t words = rows * kp;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < words; i += stride) {
        const int64_t r = i / kp;
        const int w = static_cast<int>(i - r * kp);
        const float* src = sf + r * cols;
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = 4 * w + j;
            if (c < cols) word |= ue8m0_byte(__ldg(src + c)) << (8 * j);
        }
        out[i] = word;
    }
}

// Counts scales whose sign bit is set or whose mantissa is non-zero.
__global__ void pack_ue8m0_validate_kernel(const float* __restrict__ sf, int64_t n, int32_t* __restrict__ bad) {
    griddep_launch_dependents();
    griddep_wait();
    int local = 0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
        const uint32_t bits = __float_as_uint(__ldg(sf + i));
        local += ((bits >> 31) != 0u || (bits & 0x7FFFFFu) != 0u) ? 1 : 0;
    }
    local = __reduce_add_sync(0xffffffffu, local);
    if ((threadIdx.x & 31) == 0 && local != 0) atomicAdd(bad, local);
}



// ---------------------------------------------------------------------------
// Per-token FP8 quantiser ("DeepInside DeepGEMM", section 5: the activations'
// FP8 cast and scale packing belong in a dedicated kernel before the GEMM).
// Per 1x128 block of a row: amax = max(max |x|, 1e-4f); the scale is 2^e with
// e = ceil(log2(amax / 448)), taken from the fp32 bits of amax as
// E - 8 + (mantissa > 1.75) with amax = mantissa * 2^E; the codes are
// E4M3(x * 2^-e) rounded to nearest even (|x * 2^-e| <= 448). The scale's UE8M0 byte 127 + e goes
// straight into the packed int32 scale row (byte j of word i is block
// 4i + j; the unused bytes of a row's last word are zeroed).
// One warp handles QUANT_UNROLL blocks per step, lane l taking elements
// 4l..4l+3 of each, with all their loads in flight before any use; the grid
// is QUANT_BLOCKS_PER_SM resident 256-thread blocks per SM.

// blocks per warp step: the same bytes in flight for both input types
template <bool IN_F32>
__host__ __device__ constexpr int quant_unroll() { return IN_F32 ? 8 : 16; }
constexpr int QUANT_UNROLL = 8;  // the smaller of the two (grid sizing)
constexpr int QUANT_THREADS = 256;
constexpr int QUANT_BLOCKS_PER_SM = 4;

// Raw loads of a lane's four elements (kept packed until used) and their decode.
template <bool IN_F32>
struct QuantRaw {
    using T = typename std::conditional<IN_F32, float4, uint2>::type;
    T v;
    __device__ __forceinline__ void load(const void* x, int64_t e0) {
        if constexpr (IN_F32) v = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(x) + e0));
        else v = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(x) + e0));
    }
    __device__ __forceinline__ void get(float f[4]) const {
        if constexpr (IN_F32) {
            f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
        } else {
            f[0] = __uint_as_float(v.x << 16);
            f[1] = __uint_as_float(v.x & 0xFFFF0000u);
            f[2] = __uint_as_float(v.y << 16);
            f[3] = __uint_as_float(v.y & 0xFFFF0000u);
        }
    }
};

__device__ __forceinline__ uint32_t e4m3x2_rn(float hi, float lo) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;  // e4m3(hi) in bits 15..8, e4m3(lo) in bits 7..0
}

template <bool IN_F32>
__global__ void __launch_bounds__(QUANT_THREADS, QUANT_BLOCKS_PER_SM)
quantize_fp8_1x128_kernel(const void* __restrict__ x, uint32_t* __restrict__ q,
                                          uint8_t* __restrict__ sf_bytes, float* __restrict__ sf_f32, int64_t rows,
                                          int kb, int kp) {
    griddep_launch_dependents();
    griddep_wait();
    const int lane = static_cast<int>(threadIdx.x & 31u);
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t blocks = rows * kb;
    constexpr int U = quant_unroll<IN_F32>();
    for (int64_t b0 = warp0 * U; b0 < blocks; b0 += nwarps * U) {
        QuantRaw<IN_F32> raw[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (b0 + u < blocks) raw[u].load(x, (b0 + u) * 128 + 4 * lane);
        int64_t r = b0 / kb;                    // row and block column of b0, then stepped
        int j = static_cast<int>(b0 - r * kb);
        uint32_t my_byte = 0;  // lane u < U: the scale byte of block b0 + u
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t blk = b0 + u;
            if (blk >= blocks) break;
            float v[4];
            raw[u].get(v);
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) m = max(m, __float_as_uint(v[i]) & 0x7FFFFFFFu);
            m = __reduce_max_sync(0xFFFFFFFFu, m);   // |x| bit patterns order like the values
            const uint32_t ab = max(m, __float_as_uint(1e-4f));
            const int e = static_cast<int>((ab >> 23) & 0xFFu) - 127 - 8 + ((ab & 0x7FFFFFu) > 0x600000u ? 1 : 0);
            const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e, exact
            const uint32_t lo = e4m3x2_rn(v[1] * inv, v[0] * inv);
            const uint32_t hi = e4m3x2_rn(v[3] * inv, v[2] * inv);
            q[blk * 32 + lane] = lo | (hi << 16);
            if (lane == u) my_byte = static_cast<uint32_t>(127 + e);
        }
        // scales of the step's blocks, one lane each
        if (lane < U && b0 + lane < blocks) {
            const int jj = j + lane;
            const int64_t rr = r + jj / kb;
            const int jb = jj % kb;
            uint8_t* row = sf_bytes + rr * (static_cast<int64_t>(kp) * 4);
            row[jb] = static_cast<uint8_t>(my_byte);
            if (sf_f32 != nullptr) sf_f32[b0 + lane] = __uint_as_float(my_byte << 23);
            if (jb == kb - 1)
                for (int pj = kb; pj < 4 * kp; ++pj) row[pj] = 0;
        }
    }
}

}  // namespace dg
