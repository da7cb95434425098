// kda_tile.cuh -- operand-tile addressing and the unit-lower-triangular
// inverse shared by the chunked prefill kernels (kda_chunk.cu, kda_chunk2.cu).
#pragma once
#include <cstdint>

#include "kda_common.cuh"
#include "sm100.cuh"

namespace kda {

// Element (row, k) of a K-major, 128-byte-swizzled operand tile at byte
// offset `base` of `smem` whose K-blocks (32 elements of K) are `kb` bytes apart.
__device__ __forceinline__ float* K_at(uint8_t* smem, uint32_t base, uint32_t kb, int row, int k) {
    return reinterpret_cast<float*>(smem + base + (k >> 5) * kb + sw128_off(row, (k & 31) >> 2)) + (k & 3);
}

// Byte offset of element (row, k) inside such a tile (for tiles in global memory).
__device__ __forceinline__ uint32_t K_off(uint32_t kb, int row, int k) {
    return (k >> 5) * kb + sw128_off(row, (k & 31) >> 2) + 4u * (k & 3);
}

__device__ __forceinline__ float4 tf32x4(float a, float b, float c, float d) {
    return make_float4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}

__device__ __forceinline__ void st_tf32x4(uint8_t* smem, uint32_t off, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(smem + off) = tf32x4(a, b, c, d);
}

// Barrier over a subset of the block's warps (ids 1..15; id 0 is __syncthreads).
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// TMEM address of lane quarter `quarter` (lanes 32*quarter ..), column `col`.
__device__ __forceinline__ uint32_t tm_lane(uint32_t tmem, int quarter, uint32_t col) {
    return tmem + (static_cast<uint32_t>(32 * quarter) << 16) + col;
}

// Descriptor of a K-major SW128 tile at byte offset `base` of shared memory `sb`.
__device__ __forceinline__ uint64_t tdesc(uint32_t sb, uint32_t base) { return sdesc_sw128(sb + base, 16, 1024); }

// mma.sync fragments from plain row-major fp32 arrays (leading dimension ld),
// rounded to tf32 on the way: A tile 16 x 8 at (r0, k0), B tile 8 x 8 at (k0, n0).
__device__ __forceinline__ void frag_a(uint32_t (&a)[4], const float* X, int ld, int r0, int k0, int g, int t) {
    a[0] = tf32_bits(X[(r0 + g) * ld + k0 + t]);
    a[1] = tf32_bits(X[(r0 + g + 8) * ld + k0 + t]);
    a[2] = tf32_bits(X[(r0 + g) * ld + k0 + t + 4]);
    a[3] = tf32_bits(X[(r0 + g + 8) * ld + k0 + t + 4]);
}
__device__ __forceinline__ void frag_b(uint32_t (&b)[2], const float* Y, int ld, int k0, int n0, int g, int t) {
    b[0] = tf32_bits(Y[(k0 + t) * ld + n0 + g]);
    b[1] = tf32_bits(Y[(k0 + t + 4) * ld + n0 + g]);
}
__device__ __forceinline__ void frag_store(float* D, int ld, int r0, int n0, const float (&d)[4], float sgn, int g,
                                           int t) {
    *reinterpret_cast<float2*>(D + (r0 + g) * ld + n0 + 2 * t) = make_float2(sgn * d[0], sgn * d[1]);
    *reinterpret_cast<float2*>(D + (r0 + g + 8) * ld + n0 + 2 * t) = make_float2(sgn * d[2], sgn * d[3]);
}

// Scratch of the triangular inverse: plain fp32 arrays with padded rows so
// column walks spread over banks.  M and T are 64 x kLd; Y1 is 2 x 16 x kLd1,
// Y2 32 x kLd2 (block-merge temporaries).
constexpr int kLd = 68, kLd1 = 20, kLd2 = 36;
constexpr uint32_t kUtScratchBytes = (2 * 64 * kLd + 2 * 16 * kLd1 + 32 * kLd2) * 4;

// T = (I + M)^-1 for a strictly lower triangular 64 x 64 M (row-major, ld kLd)
// into Tf (T is unit lower triangular; only its lower triangle and the
// diagonal blocks' upper zeros are written -- the caller masks the upper part
// when it reads T).  By blocks: the four 16 x 16 diagonal blocks by forward
// substitution (64 threads, one column each), then the 16 -> 32 merge
// T_ab = -T_aa M_ab T_bb for (a, b) = (1, 0), (3, 2), then the 32 -> 64 merge
// T_hl = -T_hh M_hl T_ll, both on mma.sync tf32 with fp32 accumulation.
// Must be called by all 256 threads of the block; contains block barriers
// (none at entry, one at exit).  Threads 128-255 run side() during the first
// phase (work independent of M and T).
template <class SideWork>
__device__ __forceinline__ void ut_inverse64(const float* Mf, float* Tf, float* Y1, float* Y2, int tid,
                                             SideWork side) {
    const int warp = tid >> 5, lane = tid & 31;
    if (tid < 64) {   // diagonal 16 x 16 blocks: column j of block b by substitution
        const int b = tid >> 4, j = tid & 15;
        const float* Mb = Mf + 16 * b * kLd + 16 * b;
        float xv[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float s0v = (r == j) ? 1.f : 0.f, s1v = 0.f;
#pragma unroll
            for (int i = 0; i < r; i += 2) {
                s0v = fmaf(-Mb[r * kLd + i], xv[i], s0v);
                if (i + 1 < r) s1v = fmaf(-Mb[r * kLd + i + 1], xv[i + 1], s1v);
            }
            xv[r] = s0v + s1v;
        }
        float* Tb = Tf + 16 * b * kLd + 16 * b + j;
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[r * kLd] = xv[r];
    } else if (tid < 128) {   // zero blocks (0,1) and (2,3), read by the 32 -> 64 merge
        const int e = tid - 64, blk = e >> 5, rr = (e & 31) >> 1, c8 = (e & 1) * 8;
        float* z = Tf + (32 * blk + rr) * kLd + 32 * blk + 16 + c8;
        *reinterpret_cast<float4*>(z) = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(z + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
        side();
    }
    __syncthreads();
    const int gq = lane >> 2, tq = lane & 3;
    {   // 16 -> 32: warp w < 4 owns pair p = w / 2, output columns 8 (w % 2) .. +7
        const int p = warp >> 1, nt = warp & 1, a = 2 * p + 1, b = 2 * p;
        if (warp < 4) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                uint32_t fa[4], fb[2];
                frag_a(fa, Mf, kLd, 16 * a, 16 * b + 8 * ks, gq, tq);
                frag_b(fb, Tf, kLd, 16 * b + 8 * ks, 16 * b + 8 * nt, gq, tq);
                mma_m16n8k8_tf32(d, fa, fb);
            }
            frag_store(Y1 + p * 16 * kLd1, kLd1, 0, 8 * nt, d, 1.f, gq, tq);
        }
        __syncthreads();
        if (warp < 4) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                uint32_t fa[4], fb[2];
                frag_a(fa, Tf, kLd, 16 * a, 16 * a + 8 * ks, gq, tq);
                frag_b(fb, Y1 + p * 16 * kLd1, kLd1, 8 * ks, 8 * nt, gq, tq);
                mma_m16n8k8_tf32(d, fa, fb);
            }
            frag_store(Tf, kLd, 16 * a, 16 * b + 8 * nt, d, -1.f, gq, tq);
        }
    }
    __syncthreads();
    {   // 32 -> 64: warp w owns the 16 x 8 output tile (rows 16 (w / 4), columns 8 (w % 4))
        const int mt = warp >> 2, nt = warp & 3;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t fa[4], fb[2];
            frag_a(fa, Mf, kLd, 32 + 16 * mt, 8 * ks, gq, tq);
            frag_b(fb, Tf, kLd, 8 * ks, 8 * nt, gq, tq);
            mma_m16n8k8_tf32(d, fa, fb);
        }
        frag_store(Y2, kLd2, 16 * mt, 8 * nt, d, 1.f, gq, tq);
        __syncthreads();
        float e4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t fa[4], fb[2];
            frag_a(fa, Tf, kLd, 32 + 16 * mt, 32 + 8 * ks, gq, tq);
            frag_b(fb, Y2, kLd2, 8 * ks, 8 * nt, gq, tq);
            mma_m16n8k8_tf32(e4, fa, fb);
        }
        frag_store(Tf, kLd, 32 + 16 * mt, 8 * nt, e4, -1.f, gq, tq);
    }
    __syncthreads();
}

// Prep of one chunk of up to 64 tokens, for the calling thread's 8 token rows
// r = 8 * warp + m (m = 0..7) and 4 channels 4 * lane .. 4 * lane + 3:
//   Gamma_r = g_0 + ... + g_r per channel (log2 units), Gamma_C = Gamma_63
//   (rows past L carry g = 0, so Gamma_C is the value at the last token);
//   q^, k^ = L2-normalised rows (if l2norm), then
//   Kt = k^ 2^(Gamma_r - Gamma_C),  Qt = scale q^ 2^(Gamma_r - Gamma_C),
//   Kb = k^ 2^(Gamma_C - Gamma_r),  all zero for rows r >= L.
// greg holds the thread's g values (rows x channels, natural-log units);
// rq / rk point at the raw bf16 q / k rows ([64][128]), which are read into
// registers before the block barrier inside, so emit may overwrite them.
// emit(r, kbi, ch, kt, qt, kb) receives the fp32 values of row r for the
// K-block kbi = lane / 8 and 16-byte chunk ch = lane % 8 of a K-major tile.
// gc receives Gamma_C (log2 units) of the thread's 4 channels.  xch is a
// shared [8][128] exchange buffer.  All 256 threads must call it.
template <class Emit>
__device__ __forceinline__ void prep_chunk_rows(const uint8_t* rq, const uint8_t* rk, const float (&greg)[8][4],
                                                float* xch, int L, float scale, bool l2norm, float2 (&gc)[2],
                                                Emit emit) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint2 qraw[8], kraw[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int r = 8 * warp + m;
        qraw[m] = *reinterpret_cast<const uint2*>(rq + r * kD * 2 + lane * 8);
        kraw[m] = *reinterpret_cast<const uint2*>(rk + r * kD * 2 + lane * 8);
    }
    // Gamma as channel pairs: prefix over the thread's 8 rows, then over warps
    // through shared memory
    const float2 l2e = make_float2(kLog2e, kLog2e);
    float2 G[8][2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        float2 run = make_float2(0.f, 0.f);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            run = __ffma2_rn(make_float2(greg[m][2 * x], greg[m][2 * x + 1]), l2e, run);
            G[m][x] = run;
        }
        *reinterpret_cast<float2*>(xch + warp * 128 + 4 * lane + 2 * x) = run;
    }
    __syncthreads();   // also: every thread holds its raw q, k in registers
    float2 off[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    gc[0] = gc[1] = make_float2(0.f, 0.f);
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const float4 t = *reinterpret_cast<const float4*>(xch + w * 128 + 4 * lane);
        if (w < warp) {
            off[0] = __fadd2_rn(off[0], make_float2(t.x, t.y));
            off[1] = __fadd2_rn(off[1], make_float2(t.z, t.w));
        }
        gc[0] = __fadd2_rn(gc[0], make_float2(t.x, t.y));
        gc[1] = __fadd2_rn(gc[1], make_float2(t.z, t.w));
    }
    // offset to the chunk end: Gamma_r - Gamma_C = G + (off - gc)
    const float2 rel[2] = {__fadd2_rn(off[0], make_float2(-gc[0].x, -gc[0].y)),
                           __fadd2_rn(off[1], make_float2(-gc[1].x, -gc[1].y))};

    // unpack, mask rows past the sequence end, and L2-normalise all 8 rows
    float2 qv[8][2], kv[8][2];
    float nrm[16];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const bool live = 8 * warp + m < L;
        qv[m][0] = make_float2(__uint_as_float(qraw[m].x << 16), __uint_as_float(qraw[m].x & 0xFFFF0000u));
        qv[m][1] = make_float2(__uint_as_float(qraw[m].y << 16), __uint_as_float(qraw[m].y & 0xFFFF0000u));
        kv[m][0] = make_float2(__uint_as_float(kraw[m].x << 16), __uint_as_float(kraw[m].x & 0xFFFF0000u));
        kv[m][1] = make_float2(__uint_as_float(kraw[m].y << 16), __uint_as_float(kraw[m].y & 0xFFFF0000u));
        if (!live) {
            qv[m][0] = qv[m][1] = kv[m][0] = kv[m][1] = make_float2(0.f, 0.f);
        }
        const float2 sq = __ffma2_rn(qv[m][1], qv[m][1], __fmul2_rn(qv[m][0], qv[m][0]));
        const float2 sk = __ffma2_rn(kv[m][1], kv[m][1], __fmul2_rn(kv[m][0], kv[m][0]));
        nrm[m] = sq.x + sq.y;
        nrm[8 + m] = sk.x + sk.y;
    }
    if (l2norm) warp_allreduce16(nrm);
    const int kbi = lane >> 3, ch = lane & 7;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int r = 8 * warp + m;
        const float nq = (l2norm ? rsqrtf(nrm[m] + kNormEps) : 1.f) * scale;
        const float nk = l2norm ? rsqrtf(nrm[8 + m] + kNormEps) : 1.f;
        float4 kt, qt, kb;
        float* ktp = &kt.x;
        float* qtp = &qt.x;
        float* kbp = &kb.x;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            // a = (Gamma_r - Gamma_C) / ln 2 >= 0 (the decay is cumulative, g <= 0)
            const float2 a = __fadd2_rn(G[m][x], rel[x]);
            const float2 e = make_float2(ex2(fminf(a.x, 126.f)), ex2(fminf(a.y, 126.f)));   // E >= 1
            const float2 f = make_float2(ex2(-a.x), ex2(-a.y));                              // F <= 1
            const float2 kn = __fmul2_rn(kv[m][x], make_float2(nk, nk));
            const float2 qn = __fmul2_rn(qv[m][x], make_float2(nq, nq));
            const float2 t1 = __fmul2_rn(kn, e), t2 = __fmul2_rn(qn, e), t3 = __fmul2_rn(kn, f);
            ktp[2 * x] = t1.x; ktp[2 * x + 1] = t1.y;
            qtp[2 * x] = t2.x; qtp[2 * x + 1] = t2.y;
            kbp[2 * x] = t3.x; kbp[2 * x + 1] = t3.y;
        }
        emit(r, kbi, ch, kt, qt, kb);
    }
}

}  // namespace kda
