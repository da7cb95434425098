// kda_common.cuh -- small shared helpers of the KDA CUDA kernels.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace kda {

constexpr int kD = 128;            // head dimension (d_k = d_v)
constexpr float kNormEps = 1e-6f;  // q/k L2-normalisation epsilon
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Load 4 consecutive elements (16-byte aligned for fp32, 8-byte for bf16) as fp32.
__device__ __forceinline__ void load4(const float* p, float (&r)[4]) {
    float4 v = *reinterpret_cast<const float4*>(p);
    r[0] = v.x; r[1] = v.y; r[2] = v.z; r[3] = v.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&r)[4]) {
    uint2 v = *reinterpret_cast<const uint2*>(p);
    r[0] = __uint_as_float(v.x << 16);
    r[1] = __uint_as_float(v.x & 0xFFFF0000u);
    r[2] = __uint_as_float(v.y << 16);
    r[3] = __uint_as_float(v.y & 0xFFFF0000u);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Device-side error word (first 32-bit word of the prefill workspace).
__device__ __forceinline__ void set_error(uint32_t* err, uint32_t bit) {
    if (err) atomicOr(err, bit);
}

}  // namespace kda
