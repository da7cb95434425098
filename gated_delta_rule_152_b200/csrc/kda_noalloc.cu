// kda_noalloc.cu -- kda_chunk_fwd_noalloc: the prefill call for callers that
// cannot allocate device memory.
//
// Some callers cannot hand the library a workspace: code that runs where
// cudaMalloc is forbidden or unsafe (inside a custom allocator's own callbacks,
// in an embedding runtime that owns every byte of device memory, or in a
// process that must not allocate after start-up).  For them this entry point
// uses a scratch buffer that lives inside the library itself: a file-scope
// __device__ array of kNoAllocScratchBytes bytes.  Every GPU that loads the
// library holds that array until the process exits.  The array holds the
// error word and the per-sequence reserve (kda_chunk_fwd_workspace_size_min),
// not the per-chunk scratch of the two-pass path, so bf16 prefill through
// this entry point runs the fused single kernel.
//
// The array's host-side name is only a stand-in for the symbol, not a device
// address, so the device address is looked up with cudaGetSymbolAddress, once
// per device, with that device current, the first time this entry point runs
// on it.  That first call should therefore happen before any stream capture.
// All calls share the one array and it keeps the previous call's contents:
// the error word is cleared at the start of every call, and calls whose work
// overlaps on the GPU (different streams without ordering, or several host
// threads) race on it.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/kda.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 64 * 1024;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_kda_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" KDA_API int kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g,
                                             const float* beta, const int32_t* cu_seqlens, int32_t N,
                                             int64_t total_T, int32_t H, int32_t d, kda_dtype dt,
                                             float scale, uint32_t flags, const float* initial_state,
                                             float* final_state, float* o, kda_stream_t stream) {
    const size_t need = kda_chunk_fwd_workspace_size_min(N, total_T, H, d, dt);
    if (need == 0) return d != 128 ? KDA_ERR_UNSUPPORTED : KDA_ERR_INVALID_ARG;
    if (need > kNoAllocScratchBytes) return KDA_ERR_WORKSPACE;   // N above KDA_NOALLOC_MAX_SEQS

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return KDA_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (g_scratch_addr[dev] == nullptr) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_kda_noalloc_scratch) != cudaSuccess || p == nullptr)
                return KDA_ERR_CUDA;
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }
    return kda_chunk_fwd(q, k, v, g, beta, cu_seqlens, N, total_T, H, d, dt, scale, flags, initial_state,
                         final_state, o, scratch, kNoAllocScratchBytes, stream);
}
