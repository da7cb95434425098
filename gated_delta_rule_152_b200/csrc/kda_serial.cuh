// kda_serial.cuh -- the token-by-token KDA recurrence in fp32 on CUDA cores for
// one (sequence, head, 32-column value slice), as a block-level routine shared
// by the recurrent kernel (kda_recurrent.cu) and the fused chunked kernel
// (kda_chunk.cu), which falls back to it for a sequence whose decay is too
// strong for its single reference point per chunk.
//
// The update rule of page "GLM-5.3-FLASH" (dimsnsums.com), section "How can a
// layer remember without rereading?":
//     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
//     o_t = scale * S_t^T q_t,
// one token after the other, in the expanded form
//     S' = Diag(alpha) S,  u = S'^T k,  S = S' + beta k (v - u)^T,  o = S^T q.
//
// Run by 128 threads (4 warps; thread 32 w + l owns state column
// j = 32 slice + l and key rows 32 w .. 32 w + 31 in registers).  The two
// reductions over key rows per token (u and o) combine the four warps'
// partial sums through shared memory.  Inputs are staged 16 tokens at a time.
// Synchronises with named barrier `bar_id` over those 128 threads only.
#pragma once
#include <cstdint>

#include "kda_common.cuh"

namespace kda {

constexpr int kSerialTB = 16;      // tokens staged per pass
constexpr int kSerialSlice = 32;   // value columns per slice
// Shared memory of serial_slice, in floats: K, Q, alpha [16][128]; V [16][32];
// beta [16]; the two reduction buffers [2][4][32].
constexpr int kSerialSmemFloats = 3 * kSerialTB * kD + kSerialTB * kSerialSlice + kSerialTB + 2 * 2 * 4 * kSerialSlice;

template <typename T>
__device__ __forceinline__ void serial_slice(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                                             const float* __restrict__ g, const float* __restrict__ beta,
                                             int64_t bos, int64_t eos, int H, int h, int slice, float scale,
                                             bool l2norm, bool scalar_g, const float* s0, float* sT,
                                             size_t state_off, float* __restrict__ o, float* __restrict__ snap,
                                             float* sm, int t, uint32_t bar_id) {
    float(*Ks)[kD] = reinterpret_cast<float(*)[kD]>(sm);
    float(*Qs)[kD] = reinterpret_cast<float(*)[kD]>(sm + kSerialTB * kD);
    float(*As)[kD] = reinterpret_cast<float(*)[kD]>(sm + 2 * kSerialTB * kD);
    float(*Vs)[kSerialSlice] = reinterpret_cast<float(*)[kSerialSlice]>(sm + 3 * kSerialTB * kD);
    float* Bs = sm + 3 * kSerialTB * kD + kSerialTB * kSerialSlice;
    float(*red_u)[4][kSerialSlice] = reinterpret_cast<float(*)[4][kSerialSlice]>(Bs + kSerialTB);
    float(*red_o)[4][kSerialSlice] = red_u + 2;
    auto sync = [&]() { asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory"); };

    const int warp = t >> 5, lane = t & 31;
    const int col = slice * kSerialSlice + lane;
    float s[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) s[i] = s0 ? s0[state_off + (size_t)(warp * 32 + i) * kD + col] : 0.f;

    for (int64_t t0 = bos; t0 < eos; t0 += kSerialTB) {
        const int L = (int)(eos - t0 < kSerialTB ? eos - t0 : (int64_t)kSerialTB);
        sync();   // previous pass finished reading the staged tokens
        // stage raw q, k, alpha = exp(g) for L tokens (4 channels per thread per token)
        for (int e = t; e < kSerialTB * (kD / 4); e += 128) {
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
        for (int e = t; e < kSerialTB * kSerialSlice; e += 128) {
            const int tt = e / kSerialSlice, c = e % kSerialSlice;
            Vs[tt][c] = tt < L ? to_f32(v[((size_t)(t0 + tt) * H + h) * kD + slice * kSerialSlice + c]) : 0.f;
        }
        if (t < kSerialTB) Bs[t] = t < L ? beta[(t0 + t) * H + h] : 0.f;
        sync();
        if (l2norm) {   // warp w normalises tokens w, w+4, w+8, w+12
            for (int tt = warp; tt < kSerialTB; tt += 4) {
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
            sync();
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
            sync();
            u = red_u[buf][0][lane] + red_u[buf][1][lane] + red_u[buf][2][lane] + red_u[buf][3][lane];
            const float delta = Bs[tt] * (Vs[tt][lane] - u);
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                s[i] = fmaf(Ks[tt][warp * 32 + i], delta, s[i]);
                acc = fmaf(s[i], Qs[tt][warp * 32 + i], acc);
            }
            red_o[buf][warp][lane] = acc;
            sync();
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

}  // namespace kda
