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

// Per-thread channel data of one chunk, for the calling thread's 4 channels
// 4 * lane .. 4 * lane + 3 (every warp holds the same values): rho[a] is the
// cumulative log-decay Gamma (log2 units, relative to the chunk start, so
// <= 0) at the last token of the 16-token block a; rho[3] = Gamma_C.
struct ChunkChannels {
    float4 rho[4];
    float4 bstart, bend;   // Gamma before and after the 16-token block of the thread's rows
};

// Largest exponent (log2 units) one factor of a factorised decay product may
// carry: 2^100 and 2^-100 are far inside the fp32 / tf32 normal range, so
// neither overflow nor flushed subnormals can occur below it.
constexpr float kSafeLog2 = 100.f;

// How the intra-chunk Gram matrices A_ri = sum_c k_rc k_ic 2^(Gamma_rc - Gamma_ic)
// and P (same with q_r) of a chunk are taken, by the decay it carries:
//   0: every channel decays by at most kSafeLog2 over the chunk -- one
//      tensor-core product through the chunk end, (x 2^(Gamma_r - Gamma_C))
//      (k 2^(Gamma_C - Gamma_i))^T;
//   1: every channel decays by at most kSafeLog2 inside each 16-token block --
//      block references: with rho_a the chunk's Gamma at the end of block a
//      (rho_-1 = 0), X_r = 2^(Gamma_r - rho_{a(r)-1}), Y_i = 2^(rho_{b(i)} - Gamma_i)
//      and Z_ab = 2^(rho_{a-1} - rho_b) for blocks b <= a,
//      2^(Gamma_r - Gamma_i) = X_r Z_{a(r) b(i)} Y_i, where X, Y, Z_ab (b < a)
//      lie in (0, 1] and Z_aa <= 2^kSafeLog2;
//   2: otherwise -- the same for pairs of different blocks, and every
//      2^(Gamma_r - Gamma_i) inside a block on its own.
// All three reproduce the per-token rule exactly up to rounding.

// Prep of one chunk of up to 64 tokens, for the calling thread's 8 token rows
// r = 8 * warp + m (m = 0..7, all inside 16-token block warp / 2) and 4
// channels 4 * lane .. 4 * lane + 3:
//   Gamma_r = g_0 + ... + g_r per channel (log2 units; rows past the chunk's
//   last token carry g = 0, so Gamma_C = Gamma_63 is the value at its last
//   token); q^, k^ = L2-normalised rows (if l2norm), q^ scaled by `scale`,
//   zero for r >= L.
// greg holds the thread's g values (rows x channels, natural-log units);
// rq / rk point at the raw bf16 q / k rows ([64][128]), which are read into
// registers before the block barrier inside, so emit may overwrite them.
// Calls setup(cc, level) once, with the block ends of the thread's channels
// and the chunk's Gram level (the same in every thread of the block), then
// emit(r, kbi, ch, qn, kn, gr) with the fp32 q^, k^ and Gamma_r of row r for
// the K-block kbi = lane / 8 and 16-byte chunk ch = lane % 8 of a K-major
// tile.  Returns the level.  xch is a shared [8][128] exchange buffer.  All
// 256 threads must call it.  With kMaxLevel < 2 and a chunk of a higher level,
// it returns after setup without calling emit (the raw rows are then still in
// place; a block barrier must separate this call from the next one).
template <int kMaxLevel = 2, class Setup, class Emit>
__device__ __forceinline__ int prep_chunk_rows(const uint8_t* rq, const uint8_t* rk, const float (&greg)[8][4],
                                               float* xch, int L, float scale, bool l2norm, Setup setup,
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
    // off = Gamma before this warp's first row; a block ends every second warp
    ChunkChannels cc;
    float2 run[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float2 off[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const float4 t = *reinterpret_cast<const float4*>(xch + w * 128 + 4 * lane);
        if (w == warp) {
            off[0] = run[0];
            off[1] = run[1];
        }
        if (w == (warp & 6)) cc.bstart = make_float4(run[0].x, run[0].y, run[1].x, run[1].y);
        run[0] = __fadd2_rn(run[0], make_float2(t.x, t.y));
        run[1] = __fadd2_rn(run[1], make_float2(t.z, t.w));
        if (w & 1) cc.rho[w >> 1] = make_float4(run[0].x, run[0].y, run[1].x, run[1].y);
        if (w == (warp | 1)) cc.bend = make_float4(run[0].x, run[0].y, run[1].x, run[1].y);
    }
    // the Gram level: every warp holds the same per-lane data, so the vote is block-uniform
    float block_decay = 0.f;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const float4 pr = a ? cc.rho[a - 1] : make_float4(0.f, 0.f, 0.f, 0.f), c = cc.rho[a];
        block_decay = fmaxf(block_decay, fmaxf(fmaxf(pr.x - c.x, pr.y - c.y), fmaxf(pr.z - c.z, pr.w - c.w)));
    }
    const float chunk_decay = fmaxf(fmaxf(-cc.rho[3].x, -cc.rho[3].y), fmaxf(-cc.rho[3].z, -cc.rho[3].w));
    const int level = !__any_sync(0xffffffffu, chunk_decay > kSafeLog2)   ? 0
                      : !__any_sync(0xffffffffu, block_decay > kSafeLog2) ? 1
                                                                          : 2;
    setup(cc, level);
    if (kMaxLevel < 2 && level > kMaxLevel) return level;

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
        const float2 q0 = __fmul2_rn(qv[m][0], make_float2(nq, nq)), q1 = __fmul2_rn(qv[m][1], make_float2(nq, nq));
        const float2 k0 = __fmul2_rn(kv[m][0], make_float2(nk, nk)), k1 = __fmul2_rn(kv[m][1], make_float2(nk, nk));
        const float2 g0 = __fadd2_rn(G[m][0], off[0]), g1 = __fadd2_rn(G[m][1], off[1]);
        emit(r, kbi, ch, make_float4(q0.x, q0.y, q1.x, q1.y), make_float4(k0.x, k0.y, k1.x, k1.y),
             make_float4(g0.x, g0.y, g1.x, g1.y));
    }
    return level;
}

__device__ __forceinline__ float4 ex2x4(float4 a) { return make_float4(ex2(a.x), ex2(a.y), ex2(a.z), ex2(a.w)); }
// elementwise products and differences as pairs (one f32x2 instruction per pair)
__device__ __forceinline__ float4 mul4(float4 a, float4 b) {
    const float2 lo = __fmul2_rn(make_float2(a.x, a.y), make_float2(b.x, b.y));
    const float2 hi = __fmul2_rn(make_float2(a.z, a.w), make_float2(b.z, b.w));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}
__device__ __forceinline__ float4 sub4(float4 a, float4 b) {
    const float2 lo = __fadd2_rn(make_float2(a.x, a.y), make_float2(-b.x, -b.y));
    const float2 hi = __fadd2_rn(make_float2(a.z, a.w), make_float2(-b.z, -b.w));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// ---------------------------------------------------------------- exact Gram
// Gram matrices of a chunk at level 1 or 2, on CUDA cores and mma.sync, for
// the prep of the two-pass prefill.  Inputs (fp32, K-major 128-byte-swizzled
// tiles as the emit wrote them):
//   xt  128 rows: rows 0-63 Q-side, rows 64-127 K-side;
//   yt  64 rows;
// level 1: xt = [q^ X ; k^ X], yt = k^ Y rounded to tf32 (block references, see above);
// level 2: xt = [q^ ; k^], yt = Gamma (log2), converted here in place to the
//          level-1 tiles once the in-block pairs are done;
// rho: [4][128] block-end Gammas (shared memory);  ztab: [10][128] scratch.
// Output: the unmasked 64 x 64 matrices P (rows 0-63) and A (rows 64-127) as
// plain fp32 rows of kStLd floats in `st`, which may be xt itself (it is only
// written after every read of the inputs).  Entries above the diagonal are
// left undefined.  All 256 threads; block barriers inside (none at entry,
// one at exit).  `mid` runs once every input read is done, before the output
// is written (it may reuse yt and ztab).
constexpr int kStLd = 68;
static_assert(128 * kStLd * 4 <= 65536, "staging fits the 64 KB [Q ; K] tile");

// Block pair of mma unit u: pairs p = a (a + 1) / 2 + b in order, or at level
// 2 only those with b < a (p = 1, 3, 4, 6, 7, 8).
__device__ __forceinline__ int gram_pair(int u, int level) {
    const int p = u >> 1;
    return level == 2 ? p + 1 + (p >= 1) + (p >= 3) : p;
}

template <class Mid>
__device__ __forceinline__ void gram_exact(uint8_t* xt, uint32_t kbx, uint8_t* yt, uint32_t kby, const float* rho,
                                           float* ztab, float* st, int level, int tid, Mid mid) {
    const int warp = tid >> 5, lane = tid & 31;
    // Z table: entry p = a (a + 1) / 2 + b of the block pair (a, b), b <= a
    for (int e = tid; e < 10 * kD; e += 256) {
        const int p = e >> 7, c = e & (kD - 1);
        const int a = (p >= 1) + (p >= 3) + (p >= 6), b = p - a * (a + 1) / 2;
        const float prev = a ? rho[(a - 1) * kD + c] : 0.f;
        ztab[e] = ex2(fminf(prev - rho[b * kD + c], 126.f));
    }
    // level 2: pairs inside a 16-token block, one exponential each.  Thread
    // (block a, row j / 4, column group j % 4) sums four entries of P and A.
    float dq[4] = {0.f, 0.f, 0.f, 0.f}, dk[4] = {0.f, 0.f, 0.f, 0.f};
    const int pa = tid >> 6, prow = 16 * pa + ((tid & 63) >> 2), pcol = 16 * pa + 4 * (tid & 3);
    if (level == 2 && pcol <= prow) {
        for (int k = 0; k < kD; k += 4) {
            const float4 qr = *reinterpret_cast<const float4*>(K_at(xt, 0, kbx, prow, k));
            const float4 kr = *reinterpret_cast<const float4*>(K_at(xt, 0, kbx, 64 + prow, k));
            const float4 gr = *reinterpret_cast<const float4*>(K_at(yt, 0, kby, prow, k));
#pragma unroll
            for (int l = 0; l < 4; ++l) {
                const float4 ki = *reinterpret_cast<const float4*>(K_at(xt, 0, kbx, 64 + pcol + l, k));
                const float4 gi = *reinterpret_cast<const float4*>(K_at(yt, 0, kby, pcol + l, k));
                const float4 f = ex2x4(make_float4(fminf(gr.x - gi.x, 0.f), fminf(gr.y - gi.y, 0.f),
                                                   fminf(gr.z - gi.z, 0.f), fminf(gr.w - gi.w, 0.f)));
                const float4 w = mul4(ki, f);
                dq[l] = fmaf(qr.x, w.x, fmaf(qr.y, w.y, fmaf(qr.z, w.z, fmaf(qr.w, w.w, dq[l]))));
                dk[l] = fmaf(kr.x, w.x, fmaf(kr.y, w.y, fmaf(kr.z, w.z, fmaf(kr.w, w.w, dk[l]))));
            }
        }
    }
    __syncthreads();
    if (level == 2) {   // raw tiles -> level-1 tiles, in place
        for (int it = tid; it < 64 * (kD / 4); it += 256) {
            const int r = it >> 5, k = 4 * (it & 31), a = r >> 4;
            float4* qp = reinterpret_cast<float4*>(K_at(xt, 0, kbx, r, k));
            float4* kp = reinterpret_cast<float4*>(K_at(xt, 0, kbx, 64 + r, k));
            float4* yp = reinterpret_cast<float4*>(K_at(yt, 0, kby, r, k));
            const float4 g = *yp, kk = *kp, q = *qp;
            const float4 prev = a ? *reinterpret_cast<const float4*>(rho + (a - 1) * kD + k) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 cur = *reinterpret_cast<const float4*>(rho + a * kD + k);
            const float4 X = ex2x4(sub4(g, prev)), Y = ex2x4(sub4(cur, g));
            *qp = mul4(q, X);
            *kp = mul4(kk, X);
            const float4 ky = mul4(kk, Y);
            *yp = tf32x4(ky.x, ky.y, ky.z, ky.w);
        }
        __syncthreads();
    }
    // block pairs on mma.sync (tf32, fp32 accumulation): warp w takes the pairs
    // w and w + 8 of the list (gram_pair), both matrices of each (P from the
    // Q-side rows, A from the K-side rows), which share the K-side columns and
    // the Z factors.  Every row a lane reads has (row mod 8) = lane / 4, so
    // the swizzled chunk offsets are per-lane constants.
    const int gq = lane >> 2, tq = lane & 3;
    const int npairs = level == 2 ? 6 : 10;
    float d[2][2][2][4];   // [pair slot][matrix][column half][fragment]
    int pairs[2];
    uint32_t swz[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) swz[j] = (static_cast<uint32_t>(j ^ gq) << 4) + 4u * tq;
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
        const int q = warp + 8 * sl;
        pairs[sl] = q < npairs ? gram_pair(2 * q, level) : -1;
        if (pairs[sl] < 0) continue;
        const int p = pairs[sl];
        const int a = (p >= 1) + (p >= 3) + (p >= 6), b = p - a * (a + 1) / 2;
        const float* z = ztab + p * kD;
        const uint8_t* pq = xt + (16 * a + gq) * 128;          // Q-side row gq of block a
        const uint8_t* pk = xt + (64 + 16 * a + gq) * 128;     // K-side row
        const uint8_t* py = yt + (16 * b + gq) * 128;          // column rows of block b
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int nh = 0; nh < 2; ++nh)
#pragma unroll
                for (int x = 0; x < 4; ++x) d[sl][m][nh][x] = 0.f;
#pragma unroll 1
        for (int kbi = 0; kbi < 4; ++kbi) {
            const uint8_t* bq = pq + kbi * kbx;
            const uint8_t* bk = pk + kbi * kbx;
            const uint8_t* by = py + kbi * kby;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int k0 = 32 * kbi + 8 * j;
                const float z0 = z[k0 + tq], z1 = z[k0 + tq + 4];
                const uint32_t o0 = swz[2 * j], o1 = swz[2 * j + 1];
                uint32_t fa[2][4], fb[2][2];
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    const uint8_t* r = m ? bk : bq;
                    fa[m][0] = tf32_bits(*reinterpret_cast<const float*>(r + o0) * z0);
                    fa[m][1] = tf32_bits(*reinterpret_cast<const float*>(r + 8 * 128 + o0) * z0);
                    fa[m][2] = tf32_bits(*reinterpret_cast<const float*>(r + o1) * z1);
                    fa[m][3] = tf32_bits(*reinterpret_cast<const float*>(r + 8 * 128 + o1) * z1);
                }
#pragma unroll
                for (int nh = 0; nh < 2; ++nh) {   // the K-side tile is stored already rounded to tf32
                    fb[nh][0] = *reinterpret_cast<const uint32_t*>(by + nh * 8 * 128 + o0);
                    fb[nh][1] = *reinterpret_cast<const uint32_t*>(by + nh * 8 * 128 + o1);
                }
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int nh = 0; nh < 2; ++nh) mma_m16n8k8_tf32(d[sl][m][nh], fa[m], fb[nh]);
            }
        }
    }
    __syncthreads();   // every input read
    mid();
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
        if (pairs[sl] < 0) continue;
        const int p = pairs[sl];
        const int a = (p >= 1) + (p >= 3) + (p >= 6), b = p - a * (a + 1) / 2;
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int nh = 0; nh < 2; ++nh) {
                const int row = 64 * m + 16 * a + gq, col = 16 * b + 8 * nh + 2 * tq;
                *reinterpret_cast<float2*>(st + row * kStLd + col) = make_float2(d[sl][m][nh][0], d[sl][m][nh][1]);
                *reinterpret_cast<float2*>(st + (row + 8) * kStLd + col) =
                    make_float2(d[sl][m][nh][2], d[sl][m][nh][3]);
            }
    }
    if (level == 2 && pcol <= prow) {
        *reinterpret_cast<float4*>(st + prow * kStLd + pcol) = make_float4(dq[0], dq[1], dq[2], dq[3]);
        *reinterpret_cast<float4*>(st + (64 + prow) * kStLd + pcol) = make_float4(dk[0], dk[1], dk[2], dk[3]);
    }
    __syncthreads();
}

}  // namespace kda
