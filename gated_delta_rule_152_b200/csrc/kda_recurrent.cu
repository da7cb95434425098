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
// Grid: one block per (sequence, head, 32-column value slice), flattened.
// Block: 128 threads = 4 warps.
// Thread (warp w, lane l) owns state column j = 32*slice + l and key rows
// 32*w .. 32*w+31 in registers.  The two reductions over key rows per token
// (u and o) combine the four warps' partial sums through shared memory.
// Inputs are staged 16 tokens at a time.
#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {
namespace {

constexpr int kTB = 16;        // tokens staged per pass
constexpr int kSlice = 32;     // value columns per CTA
constexpr int kThreads = 128;

template <typename T>
__global__ void __launch_bounds__(kThreads)
kda_recurrent_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const float* __restrict__ g, const float* __restrict__ beta,
                     const int32_t* __restrict__ cu_seqlens, int64_t total_T, int H, float scale,
                     int l2norm, int scalar_g, const float* s0, float* sT,
                     float* __restrict__ o, uint32_t* err, const int32_t* __restrict__ slots,
                     int num_slots, float* __restrict__ snap) {
    __shared__ float Ks[kTB][kD];
    __shared__ float Qs[kTB][kD];
    __shared__ float As[kTB][kD];
    __shared__ float Vs[kTB][kSlice];
    __shared__ float Bs[kTB];
    __shared__ float red_u[2][4][kSlice];
    __shared__ float red_o[2][4][kSlice];

    const int bid = blockIdx.x;
    const int slice = bid % (kD / kSlice), h = (bid / (kD / kSlice)) % H, n = bid / ((kD / kSlice) * H);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int col = slice * kSlice + lane;

    int64_t bos = cu_seqlens[n], eos = cu_seqlens[n + 1];
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
    float s[32];
#pragma unroll
    for (int i = 0; i < 32; ++i)
        s[i] = s0 ? s0[state_off + (size_t)(warp * 32 + i) * kD + col] : 0.f;

    for (int64_t t0 = bos; t0 < eos; t0 += kTB) {
        const int L = (int)(eos - t0 < kTB ? eos - t0 : (int64_t)kTB);
        __syncthreads();   // previous pass finished reading the staged tokens
        // stage raw q, k, alpha = exp(g) for L tokens (4 channels per thread per token)
        for (int e = threadIdx.x; e < kTB * (kD / 4); e += kThreads) {
            const int tt = e / (kD / 4), c4 = (e % (kD / 4)) * 4;
            float qv[4] = {0, 0, 0, 0}, kv[4] = {0, 0, 0, 0}, gv[4] = {0, 0, 0, 0};
            if (tt < L) {
                const size_t off = ((size_t)(t0 + tt) * H + h) * kD + c4;
                load4(q + off, qv);
                load4(k + off, kv);
                if (scalar_g) {
                    const float gs = g[(size_t)(t0 + tt) * H + h];
                    gv[0] = gv[1] = gv[2] = gv[3] = gs;
                } else {
                    load4(g + off, gv);
                }
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                Qs[tt][c4 + x] = qv[x];
                Ks[tt][c4 + x] = kv[x];
                As[tt][c4 + x] = expf(gv[x]);
            }
        }
        for (int e = threadIdx.x; e < kTB * kSlice; e += kThreads) {
            const int tt = e / kSlice, c = e % kSlice;
            Vs[tt][c] = tt < L ? to_f32(v[((size_t)(t0 + tt) * H + h) * kD + slice * kSlice + c]) : 0.f;
        }
        if (threadIdx.x < kTB) Bs[threadIdx.x] = threadIdx.x < L ? beta[(t0 + threadIdx.x) * H + h] : 0.f;
        __syncthreads();
        if (l2norm) {   // warp w normalises tokens w, w+4, w+8, w+12
            for (int tt = warp; tt < kTB; tt += 4) {
                float sq = 0.f, sk = 0.f;
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float a = Qs[tt][lane * 4 + x], b = Ks[tt][lane * 4 + x];
                    sq += a * a;
                    sk += b * b;
                }
                sq = warp_sum(sq);
                sk = warp_sum(sk);
                const float rq = rsqrtf(sq + kNormEps), rk = rsqrtf(sk + kNormEps);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    Qs[tt][lane * 4 + x] *= rq;
                    Ks[tt][lane * 4 + x] *= rk;
                }
            }
            __syncthreads();
        }
        for (int tt = 0; tt < L; ++tt) {
            const int buf = tt & 1;
            float u = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                s[i] *= As[tt][warp * 32 + i];
                u = fmaf(s[i], Ks[tt][warp * 32 + i], u);
            }
            red_u[buf][warp][lane] = u;
            __syncthreads();
            u = red_u[buf][0][lane] + red_u[buf][1][lane] + red_u[buf][2][lane] + red_u[buf][3][lane];
            const float delta = Bs[tt] * (Vs[tt][lane] - u);
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                s[i] = fmaf(Ks[tt][warp * 32 + i], delta, s[i]);
                acc = fmaf(s[i], Qs[tt][warp * 32 + i], acc);
            }
            red_o[buf][warp][lane] = acc;
            __syncthreads();
            if (warp == 0) {
                const float ov = red_o[buf][0][lane] + red_o[buf][1][lane] + red_o[buf][2][lane] +
                                 red_o[buf][3][lane];
                o[((size_t)(t0 + tt) * H + h) * kD + col] = scale * ov;
            }
            if (snap) {   // state after this token (one coalesced 128-byte row segment per store)
                float* dst = snap + ((size_t)(t0 + tt) * H + h) * kD * kD + (size_t)(warp * 32) * kD + col;
#pragma unroll
                for (int i = 0; i < 32; ++i) dst[(size_t)i * kD] = s[i];
            }
        }
    }
    if (sT) {
#pragma unroll
        for (int i = 0; i < 32; ++i) sT[state_off + (size_t)(warp * 32 + i) * kD + col] = s[i];
    }
}

}  // namespace

cudaError_t launch_recurrent(const PrefillArgs& a, cudaStream_t stream) {
    const unsigned grid = static_cast<unsigned>((long long)a.N * a.H * (kD / kSlice));
    if (a.bf16)
        kda_recurrent_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
            static_cast<const __nv_bfloat16*>(a.v), a.g, a.beta, a.cu_seqlens, a.total_T, a.H,
            a.scale, a.l2norm ? 1 : 0, a.scalar_decay ? 1 : 0, a.initial_state, a.final_state, a.o, a.err,
            a.slots, a.num_slots, a.snapshots);
    else
        kda_recurrent_kernel<float><<<grid, kThreads, 0, stream>>>(
            static_cast<const float*>(a.q), static_cast<const float*>(a.k),
            static_cast<const float*>(a.v), a.g, a.beta, a.cu_seqlens, a.total_T, a.H, a.scale,
            a.l2norm ? 1 : 0, a.scalar_decay ? 1 : 0, a.initial_state, a.final_state, a.o, a.err, a.slots,
            a.num_slots, a.snapshots);
    return cudaGetLastError();
}

}  // namespace kda
