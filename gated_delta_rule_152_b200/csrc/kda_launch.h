// kda_launch.h -- host-side launchers of the KDA kernels (internal to libkda).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace kda {

struct PrefillArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    const int32_t* cu_seqlens;
    int32_t N;
    int64_t total_T;
    int32_t H;
    bool bf16;
    float scale;
    bool l2norm;
    bool scalar_decay;   // g holds one log-decay per (token, head): [tokens, H]
    const float* initial_state;
    float* final_state;
    float* o;
    uint32_t* err;   // device error word
    const int32_t* slots = nullptr;   // optional: sequence n's state lives at index slots[n]
    int32_t num_slots = 0;            // of the state arrays (valid slots: 0 .. num_slots-1)
    float* snapshots = nullptr;       // optional [total_T, H, d, d]: the state after every token
};

// Token-by-token fp32 recurrence (CUDA cores), any dtype.
cudaError_t launch_recurrent(const PrefillArgs& a, cudaStream_t stream);

// Chunked tensor-core prefill (tcgen05, kind::tf32), bf16 q/k/v.
cudaError_t launch_chunk(const PrefillArgs& a, cudaStream_t stream);

struct DecodeArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    float* state;
    float* o;
    int32_t N;
    int32_t H;
    bool bf16;
    float scale;
    bool l2norm;
    bool scalar_decay;   // g is [N, H]
    const int32_t* slots = nullptr;   // optional: sequence n's state is state[slots[n]]
    int32_t num_slots = 0;
};

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);

}  // namespace kda
