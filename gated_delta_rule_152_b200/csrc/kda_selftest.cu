// kda_selftest.cu -- kda_selftest_bounded_waits: drives the bounded waits that
// every kernel of the library uses (a flag poll with an acquire load, an
// mbarrier try_wait loop) into their give-up path on purpose, so that tests
// can check that a wait which never completes ends with KDA_DEVERR_TIMEOUT in
// the workspace and a usable context, instead of a hang.
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/kda.h"
#include "kda_common.cuh"
#include "kda_launch.h"
#include "sm100.cuh"

namespace kda {
namespace {

__global__ void kda_selftest_kernel(uint32_t* err, const int32_t* never_set, uint32_t polls) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        // a flag nobody writes
        if (!wait_flag_ge(never_set, 1, polls)) set_error(err, 2u);
        // an mbarrier that expects one arrival that never comes
        mbar_init(&bar, 1);
        fence_mbar_init();
        if (!mbar_wait_bounded(&bar, 0, polls)) set_error(err, 2u);
    }
}

}  // namespace
}  // namespace kda

extern "C" KDA_API int kda_selftest_bounded_waits(void* workspace, size_t workspace_bytes, uint32_t polls,
                                                  kda_stream_t stream) {
    if (!workspace || workspace_bytes < 256) return KDA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return KDA_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, 8, s) != cudaSuccess) return KDA_ERR_CUDA;
    uint32_t* err = static_cast<uint32_t*>(workspace);
    return kda::launch_kernel(kda::kda_selftest_kernel, dim3(1), dim3(32), 0, s, err,
                              reinterpret_cast<const int32_t*>(err + 1), polls) == cudaSuccess
               ? KDA_OK
               : KDA_ERR_CUDA;
}
