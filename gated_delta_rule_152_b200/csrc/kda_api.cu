// kda_api.cu -- the C ABI of libkda (declared in include/kda.h): host-side
// argument checks, kernel selection and the device error word.
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/kda.h"
#include "kda_launch.h"

namespace {

constexpr size_t kWorkspaceHeader = 256;   // error word + reserved, keeps the rest aligned

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool device_is_sm100(int* status) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { *status = KDA_ERR_CUDA; return false; }
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        *status = KDA_ERR_CUDA;
        return false;
    }
    if (major != 10 || minor != 0) { *status = KDA_ERR_UNSUPPORTED; return false; }
    return true;
}

}  // namespace

extern "C" {

size_t kda_chunk_fwd_workspace_size_min(int32_t N, int64_t total_T, int32_t H, int32_t d, kda_dtype dt) {
    (void)dt;
    if (N < 0 || total_T < 0 || H <= 0 || d != 128) return 0;
    return kWorkspaceHeader + 4u * static_cast<size_t>(N);   // error word + reserved
}

size_t kda_chunk_fwd_workspace_size(int32_t N, int64_t total_T, int32_t H, int32_t d, kda_dtype dt) {
    const size_t lo = kda_chunk_fwd_workspace_size_min(N, total_T, H, d, dt);
    if (lo == 0) return 0;
    const size_t two_pass = kWorkspaceHeader + kda::two_pass_scratch_bytes(N, total_T, H);
    return two_pass > lo ? two_pass : lo;
}

}  // extern "C"

namespace {

// Shared body of kda_chunk_fwd and kda_chunk_fwd_slots.
int chunk_fwd_impl(const void* q, const void* k, const void* v, const float* g, const float* beta,
                   const int32_t* cu_seqlens, int32_t N, int64_t total_T, int32_t H, int32_t d,
                   kda_dtype dt, float scale, uint32_t flags, const float* initial_state,
                   float* final_state, float* o, void* workspace, size_t workspace_bytes,
                   kda_stream_t stream, const int32_t* slots, int32_t num_slots,
                   float* snapshots = nullptr) {
    if (N < 0 || H <= 0 || total_T < 0 || total_T >= (int64_t(1) << 31)) return KDA_ERR_INVALID_ARG;
    if (d != 128) return KDA_ERR_UNSUPPORTED;
    if (dt != KDA_DTYPE_BF16 && dt != KDA_DTYPE_FP32) return KDA_ERR_UNSUPPORTED;
    if (flags & ~uint32_t(KDA_FLAG_L2NORM_QK | KDA_FLAG_RECURRENT | KDA_FLAG_SCALAR_DECAY))
        return KDA_ERR_UNSUPPORTED;
    if (cu_seqlens == nullptr) return KDA_ERR_INVALID_ARG;
    if (total_T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, beta, initial_state, final_state, o, workspace, snapshots};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    if (workspace == nullptr || workspace_bytes < kda_chunk_fwd_workspace_size_min(N, total_T, H, d, dt))
        return KDA_ERR_WORKSPACE;
    int status = KDA_OK;
    if (!device_is_sm100(&status)) return status;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t* err = static_cast<uint32_t*>(workspace);
    if (cudaMemsetAsync(err, 0, sizeof(uint32_t), s) != cudaSuccess) return KDA_ERR_CUDA;
    if (N == 0) return KDA_OK;

    kda::PrefillArgs a{q, k, v, g, beta, cu_seqlens, N, total_T, H, dt == KDA_DTYPE_BF16, scale,
                       (flags & KDA_FLAG_L2NORM_QK) != 0, (flags & KDA_FLAG_SCALAR_DECAY) != 0,
                       initial_state, final_state, o, err, slots, num_slots, snapshots};
    const bool recurrent = (dt == KDA_DTYPE_FP32) || (flags & KDA_FLAG_RECURRENT) || total_T == 0 ||
                           snapshots != nullptr;
    // the two-pass tensor-core path when the workspace holds its scratch,
    // else the fused single kernel (same arithmetic, no scratch)
    const bool two_pass =
        !recurrent && workspace_bytes >= kWorkspaceHeader + kda::two_pass_scratch_bytes(N, total_T, H);
    cudaError_t e;
    if (recurrent) {
        e = kda::launch_recurrent(a, s);
    } else {
        e = two_pass ? kda::launch_chunk_two_pass(a, static_cast<uint8_t*>(workspace) + kWorkspaceHeader, s)
                     : cudaErrorNotSupported;
        // not enough room for the two-pass path on this device: the fused kernel
        if (e == cudaErrorNotSupported) e = kda::launch_chunk(a, s);
    }
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int decode_impl(const void* q, const void* k, const void* v, const float* g, const float* beta, float* state,
                float* o, int32_t N, int32_t H, int32_t d, kda_dtype dt, float scale, uint32_t flags,
                kda_stream_t stream, const int32_t* slots, int32_t num_slots) {
    if (N < 0 || H <= 0 || static_cast<int64_t>(N) * H >= (int64_t(1) << 31)) return KDA_ERR_INVALID_ARG;
    if (d != 128) return KDA_ERR_UNSUPPORTED;
    if (dt != KDA_DTYPE_BF16 && dt != KDA_DTYPE_FP32) return KDA_ERR_UNSUPPORTED;
    if (flags & ~uint32_t(KDA_FLAG_L2NORM_QK | KDA_FLAG_SCALAR_DECAY)) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return KDA_OK;
    if (!q || !k || !v || !g || !beta || !state || !o) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, beta, state, o};
    for (const void* p : ptrs)
        if (!aligned16(p)) return KDA_ERR_MISALIGNED;
    int status = KDA_OK;
    if (!device_is_sm100(&status)) return status;
    kda::DecodeArgs a{q, k, v, g, beta, state, o, N, H, dt == KDA_DTYPE_BF16, scale,
                      (flags & KDA_FLAG_L2NORM_QK) != 0, (flags & KDA_FLAG_SCALAR_DECAY) != 0, slots,
                      num_slots};
    return kda::launch_decode(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? KDA_OK
                                                                                         : KDA_ERR_CUDA;
}

}  // namespace

extern "C" {

int kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                  const int32_t* cu_seqlens, int32_t N, int64_t total_T, int32_t H, int32_t d,
                  kda_dtype dt, float scale, uint32_t flags, const float* initial_state,
                  float* final_state, float* o, void* workspace, size_t workspace_bytes,
                  kda_stream_t stream) {
    return chunk_fwd_impl(q, k, v, g, beta, cu_seqlens, N, total_T, H, d, dt, scale, flags, initial_state,
                          final_state, o, workspace, workspace_bytes, stream, nullptr, 0);
}

int kda_chunk_fwd_slots(const void* q, const void* k, const void* v, const float* g, const float* beta,
                        const int32_t* cu_seqlens, int32_t N, int64_t total_T, int32_t H, int32_t d,
                        kda_dtype dt, float scale, uint32_t flags, float* state_pool, const int32_t* slots,
                        int32_t num_slots, float* o, void* workspace, size_t workspace_bytes,
                        kda_stream_t stream) {
    if (!state_pool || !slots || num_slots <= 0) return KDA_ERR_INVALID_ARG;
    if (!aligned16(state_pool)) return KDA_ERR_MISALIGNED;
    return chunk_fwd_impl(q, k, v, g, beta, cu_seqlens, N, total_T, H, d, dt, scale, flags, state_pool,
                          state_pool, o, workspace, workspace_bytes, stream, slots, num_slots);
}

int kda_verify_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                   const int32_t* cu_seqlens, int32_t N, int64_t total_T, int32_t H, int32_t d,
                   kda_dtype dt, float scale, uint32_t flags, const float* initial_state,
                   float* state_snapshots, float* o, void* workspace, size_t workspace_bytes,
                   kda_stream_t stream) {
    if (total_T > 0 && state_snapshots == nullptr) return KDA_ERR_INVALID_ARG;
    return chunk_fwd_impl(q, k, v, g, beta, cu_seqlens, N, total_T, H, d, dt, scale, flags, initial_state,
                          nullptr, o, workspace, workspace_bytes, stream, nullptr, 0,
                          total_T > 0 ? state_snapshots : nullptr);
}

int kda_decode_step(const void* q, const void* k, const void* v, const float* g, const float* beta,
                    float* state, float* o, int32_t N, int32_t H, int32_t d, kda_dtype dt,
                    float scale, uint32_t flags, kda_stream_t stream) {
    return decode_impl(q, k, v, g, beta, state, o, N, H, d, dt, scale, flags, stream, nullptr, 0);
}

int kda_decode_step_slots(const void* q, const void* k, const void* v, const float* g, const float* beta,
                          float* state_pool, const int32_t* slots, int32_t num_slots, float* o, int32_t N,
                          int32_t H, int32_t d, kda_dtype dt, float scale, uint32_t flags,
                          kda_stream_t stream) {
    if (N > 0 && (!slots || num_slots <= 0)) return KDA_ERR_INVALID_ARG;
    return decode_impl(q, k, v, g, beta, state_pool, o, N, H, d, dt, scale, flags, stream, slots, num_slots);
}

int kda_workspace_error(const void* workspace, uint32_t* out, kda_stream_t stream) {
    if (!workspace || !out) return KDA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(out, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return KDA_ERR_CUDA;
    return cudaStreamSynchronize(s) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

const char* kda_status_string(int status) {
    switch (status) {
        case KDA_OK: return "ok";
        case KDA_ERR_INVALID_ARG: return "invalid argument";
        case KDA_ERR_UNSUPPORTED: return "unsupported size, dtype, flag or device";
        case KDA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case KDA_ERR_WORKSPACE: return "workspace missing or too small";
        case KDA_ERR_CUDA: return "CUDA error";
        default: return "unknown status";
    }
}

}  // extern "C"
