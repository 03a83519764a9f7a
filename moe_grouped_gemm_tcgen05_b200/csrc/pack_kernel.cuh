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

}  // namespace dg
