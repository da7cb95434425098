// kda_recurrent.cu -- token-by-token KDA recurrence in fp32 on CUDA cores.
//
// Evaluates the update rule of page "GLM-5.3-FLASH" (dimsnsums.com), section
// "How can a layer remember without rereading?":
//     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
//     o_t = scale * S_t^T q_t,
// one token after the other, in the expanded form
//     S' = Diag(alpha) S,  u = S'^T k,  S = S' + beta k (v - u)^T,  o = S^T q.
// It is exact fp32 arithmetic (no tensor cores), so it serves fp32 inputs at
// the tight tolerance and any input when KDA_FLAG_RECURRENT is set.  It also
// serves multi-token verification: with a snapshot array it stores the state
// after every token, so a caller can roll back to any accepted prefix.
//
// Grid: one block of 128 threads per (sequence, head, 32-column value slice),
// flattened; the recurrence itself is serial_slice (kda_serial.cuh).
#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_serial.cuh"

namespace kda {
namespace {

constexpr int kThreads = 128;

template <typename T>
__global__ void __launch_bounds__(kThreads)
kda_recurrent_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const float* __restrict__ g, const float* __restrict__ beta,
                     const int32_t* __restrict__ cu_seqlens, int64_t total_T, int H, float scale,
                     int l2norm, int scalar_g, const float* s0, float* sT,
                     float* __restrict__ o, uint32_t* err, const int32_t* __restrict__ slots,
                     int num_slots, float* __restrict__ snap) {
    __shared__ __align__(16) float sm[kSerialSmemFloats];
    const int bid = blockIdx.x;
    const int slice = bid % (kD / kSerialSlice), h = (bid / (kD / kSerialSlice)) % H,
              n = bid / ((kD / kSerialSlice) * H);

    const int64_t bos = cu_seqlens[n], eos = cu_seqlens[n + 1];
    if (bos < 0 || eos < bos || eos > total_T) {
        if (threadIdx.x == 0 && slice == 0 && h == 0) set_error(err, 1u);
        return;   // inconsistent cu_seqlens: sequence skipped
    }
    const int64_t sidx = slots ? static_cast<int64_t>(slots[n]) : static_cast<int64_t>(n);
    if (slots && (sidx < 0 || sidx >= num_slots)) {
        if (threadIdx.x == 0 && slice == 0 && h == 0) set_error(err, 4u);
        return;   // slot out of range: this sequence is skipped
    }
    const size_t state_off = ((size_t)sidx * H + h) * kD * kD;
    serial_slice(q, k, v, g, beta, bos, eos, H, h, slice, scale, l2norm != 0, scalar_g != 0, s0, sT, state_off, o,
                 snap, sm, threadIdx.x, 1u);
}

}  // namespace

cudaError_t launch_recurrent(const PrefillArgs& a, cudaStream_t stream) {
    const unsigned grid = static_cast<unsigned>((long long)a.N * a.H * (kD / kSerialSlice));
    if (a.bf16)
        return launch_kernel(kda_recurrent_kernel<__nv_bfloat16>, dim3(grid), dim3(kThreads), 0, stream,
                             static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
                             static_cast<const __nv_bfloat16*>(a.v), a.g, a.beta, a.cu_seqlens, a.total_T,
                             static_cast<int>(a.H), a.scale, a.l2norm ? 1 : 0, a.scalar_decay ? 1 : 0,
                             a.initial_state, a.final_state, a.o, a.err, a.slots, static_cast<int>(a.num_slots),
                             a.snapshots);
    return launch_kernel(kda_recurrent_kernel<float>, dim3(grid), dim3(kThreads), 0, stream,
                         static_cast<const float*>(a.q), static_cast<const float*>(a.k),
                         static_cast<const float*>(a.v), a.g, a.beta, a.cu_seqlens, a.total_T, static_cast<int>(a.H),
                         a.scale, a.l2norm ? 1 : 0, a.scalar_decay ? 1 : 0, a.initial_state, a.final_state, a.o,
                         a.err, a.slots, static_cast<int>(a.num_slots), a.snapshots);
}

}  // namespace kda
