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

// All-reduce of 16 per-lane partial sums over the 32 lanes of a warp with 32
// shuffles instead of 16 x 5: four halving exchange steps leave lane L with the
// pair-sum of entry (L >> 1) & 15, one more step completes it, and 16
// broadcasts return every total to every lane.
__device__ __forceinline__ void warp_allreduce16(float (&v)[16]) {
    const unsigned lane = threadIdx.x & 31u;
    float a8[8], a4[4], a2[2];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool up = lane & 16u;
        a8[i] = (up ? v[i + 8] : v[i]) + __shfl_xor_sync(0xffffffffu, up ? v[i] : v[i + 8], 16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool up = lane & 8u;
        a4[i] = (up ? a8[i + 4] : a8[i]) + __shfl_xor_sync(0xffffffffu, up ? a8[i] : a8[i + 4], 8);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool up = lane & 4u;
        a2[i] = (up ? a4[i + 2] : a4[i]) + __shfl_xor_sync(0xffffffffu, up ? a4[i] : a4[i + 2], 4);
    }
    const bool up = lane & 2u;
    float a1 = (up ? a2[1] : a2[0]) + __shfl_xor_sync(0xffffffffu, up ? a2[0] : a2[1], 2);
    a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = __shfl_sync(0xffffffffu, a1, 2 * e);
}

// Device-side error word (first 32-bit word of the prefill workspace).
__device__ __forceinline__ void set_error(uint32_t* err, uint32_t bit) {
    if (err) atomicOr(err, bit);
}

}  // namespace kda
