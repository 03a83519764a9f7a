// Capture-safe UE8M0 pack and its optional validator.
//
// "[GH-ISSUE #414] pack_ue8m0_to_int is not CUDA Graph capture safe", Expected
// behavior: the pack is the biased-exponent byte of each fp32 scale
// ((bits >> 23), low 8 bits), four consecutive bytes per int32, little-endian;
// the value checks (sign clear, mantissa zero) belong on a separate eager path.
// Neither kernel reads a device value back to the host.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace dg {

__device__ __forceinline__ uint32_t ue8m0_byte(float x) {
    return (__float_as_uint(x) >> 23) & 0xFFu;
}

// cols % 4 == 0 and 16-byte aligned input: word i packs floats 4i..4i+3, so the
// whole tensor is one flat stream of float4 -> int32.
__global__ void pack_ue8m0_vec4_kernel(const float4* __restrict__ sf, uint32_t* __restrict__ out, int64_t words) {
    griddep_wait();
    griddep_launch_dependents();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < words; i += stride) {
        const float4 v = __ldg(sf + i);
        out[i] = ue8m0_byte(v.x) | (ue8m0_byte(v.y) << 8) | (ue8m0_byte(v.z) << 16) | (ue8m0_byte(v.w) << 24);
    }
}

// General layout: rows x cols floats -> rows x kp words, zero bytes past cols.
__global__ void pack_ue8m0_rows_kernel(const float* __restrict__ sf, uint32_t* __restrict__ out, int64_t rows,
                                       int cols, int kp) {
    griddep_wait();
    griddep_launch_dependents();
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
    griddep_wait();
    griddep_launch_dependents();
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
// E4M3(x * 2^-e) rounded to nearest even (|x * 2^-e| <= 448, so the
// saturating convert never saturates). The scale's UE8M0 byte 127 + e goes
// straight into the packed int32 scale row (byte j of word i is block
// 4i + j; the unused bytes of a row's last word are zeroed).
// One warp handles QUANT_UNROLL blocks per step, lane l taking elements
// 4l..4l+3 of each, with all their loads in flight before any use.

constexpr int QUANT_UNROLL = 4;

template <bool IN_F32>
__device__ __forceinline__ void quant_load4(const void* x, int64_t e0, float v[4]) {
    if constexpr (IN_F32) {
        const float4 t = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(x) + e0));
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else {
        const uint2 t = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(x) + e0));
        v[0] = __uint_as_float(t.x << 16);
        v[1] = __uint_as_float(t.x & 0xFFFF0000u);
        v[2] = __uint_as_float(t.y << 16);
        v[3] = __uint_as_float(t.y & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint16_t e4m3x2_rn(float hi, float lo) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;  // e4m3(hi) in bits 15..8, e4m3(lo) in bits 7..0
}

template <bool IN_F32>
__global__ void quantize_fp8_1x128_kernel(const void* __restrict__ x, uint32_t* __restrict__ q,
                                          uint8_t* __restrict__ sf_bytes, float* __restrict__ sf_f32, int64_t rows,
                                          int kb, int kp) {
    griddep_wait();
    griddep_launch_dependents();
    const int lane = static_cast<int>(threadIdx.x & 31u);
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t blocks = rows * kb;
    for (int64_t b0 = warp0 * QUANT_UNROLL; b0 < blocks; b0 += nwarps * QUANT_UNROLL) {
        float v[QUANT_UNROLL][4];
#pragma unroll
        for (int u = 0; u < QUANT_UNROLL; ++u)
            if (b0 + u < blocks) quant_load4<IN_F32>(x, (b0 + u) * 128 + 4 * lane, v[u]);
#pragma unroll
        for (int u = 0; u < QUANT_UNROLL; ++u) {
            const int64_t blk = b0 + u;
            if (blk >= blocks) break;
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) m = max(m, __float_as_uint(v[u][i]) & 0x7FFFFFFFu);
            m = __reduce_max_sync(0xFFFFFFFFu, m);   // |x| bit patterns order like the values
            const uint32_t ab = max(m, __float_as_uint(1e-4f));
            const int e = static_cast<int>((ab >> 23) & 0xFFu) - 127 - 8 + ((ab & 0x7FFFFFu) > 0x600000u ? 1 : 0);
            const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e, exact
            const uint32_t lo = e4m3x2_rn(v[u][1] * inv, v[u][0] * inv);
            const uint32_t hi = e4m3x2_rn(v[u][3] * inv, v[u][2] * inv);
            q[blk * 32 + lane] = lo | (hi << 16);
            if (lane == 0) {
                const int64_t r = blk / kb;
                const int j = static_cast<int>(blk - r * kb);
                uint8_t* row = sf_bytes + r * (static_cast<int64_t>(kp) * 4);
                row[j] = static_cast<uint8_t>(127 + e);
                if (sf_f32 != nullptr) sf_f32[blk] = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
                if (j == kb - 1)
                    for (int pj = kb; pj < 4 * kp; ++pj) row[pj] = 0;
            }
        }
    }
}

}  // namespace dg
