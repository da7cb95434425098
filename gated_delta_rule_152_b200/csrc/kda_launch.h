// kda_launch.h -- host-side launchers of the KDA kernels (internal to libkda).
#pragma once
#include <cstdint>
#include <mutex>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

namespace kda {

// Launch `kernel` with an explicit configuration and return this launch's own
// status (cudaLaunchKernelEx's return value), so that an unrelated earlier
// error left on the calling thread by other code is neither reported as ours
// nor cleared.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// One-time set-up that CUDA keeps per device (a kernel's dynamic shared-memory
// limit, for instance): run() calls fn once for each device that is current
// when it is called, and returns that first outcome on every later call.
class PerDeviceOnce {
  public:
    template <class Fn>
    cudaError_t run(Fn fn) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        std::lock_guard<std::mutex> lock(mu_);
        if (!done_[dev]) {
            err_[dev] = fn();
            done_[dev] = true;
        }
        return err_[dev];
    }

  private:
    static constexpr int kMaxDevices = 64;
    std::mutex mu_;
    bool done_[kMaxDevices] = {};
    cudaError_t err_[kMaxDevices] = {};
};

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

// Chunked tensor-core prefill (tcgen05, kind::tf32), bf16 q/k/v, one fused
// kernel per (sequence, head, 32-column value slice); needs no scratch.
cudaError_t launch_chunk(const PrefillArgs& a, cudaStream_t stream);

// Two-pass chunked prefill: a parallel pass over (chunk, head) that writes
// each chunk's state-independent operands to scratch, then a sequential pass
// per (sequence, head) that carries the state; for a single sequence both
// passes run overlapped in one cooperative launch through a ring of operand
// slots.  `scratch` (16-byte aligned) must hold two_pass_scratch_bytes(N,
// total_T, H) bytes.  Returns cudaErrorNotSupported, having launched nothing,
// when the device cannot host the overlapped launch.
size_t two_pass_scratch_bytes(int32_t N, int64_t total_T, int32_t H);
cudaError_t launch_chunk_two_pass(const PrefillArgs& a, void* scratch, cudaStream_t stream);

// [total_T, H, 128] bf16 (or fp32) viewed as a 3-D tensor (channel, head,
// token) for TMA; one box is 64 tokens x 128 channels of one head, no swizzle.
bool make_token_map(CUtensorMap* map, const void* base, int64_t total_T, int H, bool f32 = false);

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
