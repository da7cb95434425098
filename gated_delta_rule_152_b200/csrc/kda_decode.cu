// kda_decode.cu -- one-token KDA decode step, in place, HBM-bandwidth bound.
//
// For every (sequence, head) the 128 x 128 fp32 state S advances by one token
// of the update rule on page "GLM-5.3-FLASH" (dimsnsums.com), section "How can
// a layer remember without rereading?":
//     S_new = (I - beta k k^T) Diag(alpha) S + beta k v^T,  o = scale * S_new^T q.
// With S' = Diag(alpha) S this is S_new = S' + k delta^T where
// delta = beta (v - S'^T k), and S_new^T q = S'^T q + delta (k . q).  Both
// reductions over key rows, a = S'^T k and b = S'^T q, need only alpha*k and
// alpha*q against the OLD state, so the state is read once, reduced, and
// written once: 2 x 64 KiB of HBM traffic per (sequence, head) and nothing
// else of consequence (q, k, v, g, beta, o add 1.3 KB).
//
// Block: 256 threads for one (sequence, head).  Thread (warp w, lane l) holds
// the 16 rows i = w + 8m (m = 0..15) of columns 4l .. 4l+3 as 16 float4
// registers (one warp-wide 512-byte row segment per load: fully coalesced
// 128-bit accesses).  Column sums over the 8 warps go through shared memory.
#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = kD / 8;   // rows per thread

template <typename T>
__global__ void __launch_bounds__(kThreads, 2)
kda_decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const float* __restrict__ g, const float* __restrict__ beta,
                  float* __restrict__ state, float* __restrict__ o, float scale, int l2norm, int scalar_g,
                  int H, const int32_t* __restrict__ slots, int num_slots) {
    __shared__ float ak[kD], aq[kD], al[kD], kh[kD];
    __shared__ float4 red[8][2][32];
    __shared__ float qk_dot;

    const int p = blockIdx.x;          // (sequence, head) pair, row-major [N, H]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the state of sequence n sits at index n, or at slots[n] of a state pool
    size_t sp = static_cast<size_t>(p);
    if (slots) {
        const int n = p / H, h = p - n * H, slot = slots[n];
        if (slot < 0 || slot >= num_slots) {   // out-of-range slot: sequence skipped, its o marked NaN
            if (warp == 0) reinterpret_cast<float4*>(o + (size_t)p * kD)[lane] = make_float4(NAN, NAN, NAN, NAN);
            return;
        }
        sp = static_cast<size_t>(slot) * H + h;
    }
    float4* S = reinterpret_cast<float4*>(state + sp * kD * kD);

    // 1. put the whole 64 KiB state slab in flight first (streaming loads)
    float4 s[kRows];
#pragma unroll
    for (int m = 0; m < kRows; ++m) s[m] = __ldcs(S + (warp + 8 * m) * (kD / 4) + lane);

    // 2. warp 0 normalises q, k and forms alpha*k, alpha*q while the loads fly
    if (warp == 0) {
        float qv[4], kv[4], gv[4];
        load4(q + (size_t)p * kD + lane * 4, qv);
        load4(k + (size_t)p * kD + lane * 4, kv);
        if (scalar_g) {   // one decay per (sequence, head), shared by all channels
            gv[0] = gv[1] = gv[2] = gv[3] = g[p];
        } else {
            load4(g + (size_t)p * kD + lane * 4, gv);
        }
        float rq = 1.f, rk = 1.f;
        if (l2norm) {
            float sq = 0.f, sk = 0.f;
#pragma unroll
            for (int x = 0; x < 4; ++x) { sq += qv[x] * qv[x]; sk += kv[x] * kv[x]; }
            rq = rsqrtf(warp_sum(sq) + kNormEps);
            rk = rsqrtf(warp_sum(sk) + kNormEps);
        }
        float dot = 0.f;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float qn = qv[x] * rq, kn = kv[x] * rk, a = expf(gv[x]);
            ak[lane * 4 + x] = a * kn;
            aq[lane * 4 + x] = a * qn;
            al[lane * 4 + x] = a;
            kh[lane * 4 + x] = kn;
            dot += qn * kn;
        }
        dot = warp_sum(dot);
        if (lane == 0) qk_dot = dot;
    }
    __syncthreads();

    // 3. partial column sums a_j = sum_i S_ij alpha_i k_i, b_j = sum_i S_ij alpha_i q_i
    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
    for (int m = 0; m < kRows; ++m) {
        const int i = warp + 8 * m;
        const float x = ak[i], y = aq[i];
        pa.x = fmaf(s[m].x, x, pa.x); pa.y = fmaf(s[m].y, x, pa.y);
        pa.z = fmaf(s[m].z, x, pa.z); pa.w = fmaf(s[m].w, x, pa.w);
        pb.x = fmaf(s[m].x, y, pb.x); pb.y = fmaf(s[m].y, y, pb.y);
        pb.z = fmaf(s[m].z, y, pb.z); pb.w = fmaf(s[m].w, y, pb.w);
    }
    red[warp][0][lane] = pa;
    red[warp][1][lane] = pb;
    __syncthreads();
    float4 a = red[0][0][lane], b = red[0][1][lane];
#pragma unroll
    for (int w = 1; w < 8; ++w) {
        const float4 ra = red[w][0][lane], rb = red[w][1][lane];
        a.x += ra.x; a.y += ra.y; a.z += ra.z; a.w += ra.w;
        b.x += rb.x; b.y += rb.y; b.z += rb.z; b.w += rb.w;
    }

    // 4. delta = beta (v - a); o = scale (b + (q.k) delta)
    float vv[4];
    load4(v + (size_t)p * kD + lane * 4, vv);
    const float bt = beta[p];
    float4 d;
    d.x = bt * (vv[0] - a.x); d.y = bt * (vv[1] - a.y);
    d.z = bt * (vv[2] - a.z); d.w = bt * (vv[3] - a.w);
    if (warp == 0) {
        const float qk = qk_dot;
        float4 ov;
        ov.x = scale * fmaf(qk, d.x, b.x); ov.y = scale * fmaf(qk, d.y, b.y);
        ov.z = scale * fmaf(qk, d.z, b.z); ov.w = scale * fmaf(qk, d.w, b.w);
        reinterpret_cast<float4*>(o + (size_t)p * kD)[lane] = ov;
    }

    // 5. S_ij <- alpha_i S_ij + k_i delta_j, written back in place
#pragma unroll
    for (int m = 0; m < kRows; ++m) {
        const int i = warp + 8 * m;
        const float al_i = al[i], k_i = kh[i];
        float4 r;
        r.x = fmaf(al_i, s[m].x, k_i * d.x); r.y = fmaf(al_i, s[m].y, k_i * d.y);
        r.z = fmaf(al_i, s[m].z, k_i * d.z); r.w = fmaf(al_i, s[m].w, k_i * d.w);
        __stcs(S + i * (kD / 4) + lane, r);
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    const long long pairs = (long long)a.N * a.H;
    if (pairs == 0) return cudaSuccess;
    if (a.bf16)
        return launch_kernel(kda_decode_kernel<__nv_bfloat16>, dim3((unsigned)pairs), dim3(kThreads), 0, stream,
                             static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
                             static_cast<const __nv_bfloat16*>(a.v), a.g, a.beta, a.state, a.o, a.scale,
                             a.l2norm ? 1 : 0, a.scalar_decay ? 1 : 0, static_cast<int>(a.H), a.slots,
                             static_cast<int>(a.num_slots));
    return launch_kernel(kda_decode_kernel<float>, dim3((unsigned)pairs), dim3(kThreads), 0, stream,
                         static_cast<const float*>(a.q), static_cast<const float*>(a.k),
                         static_cast<const float*>(a.v), a.g, a.beta, a.state, a.o, a.scale, a.l2norm ? 1 : 0,
                         a.scalar_decay ? 1 : 0, static_cast<int>(a.H), a.slots, static_cast<int>(a.num_slots));
}

}  // namespace kda
