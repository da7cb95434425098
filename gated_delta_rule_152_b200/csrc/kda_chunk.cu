// kda_chunk.cu -- chunked KDA prefill on Blackwell tensor cores (tcgen05,
// kind::tf32, accumulators in tensor memory, q/k tiles staged by TMA).
//
// The layer's rule (page "GLM-5.3-FLASH", dimsnsums.com, section "How can a
// layer remember without rereading?"):
//     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
//     o_t = scale * S_t^T q_t.
// The page gives only this per-token rule.  This kernel evaluates exactly the
// same recurrence 64 tokens at a time.  For one chunk with entry state S
// (rows = key channels), Gamma_r = g_0 + ... + g_r per channel and
// Gamma_C = Gamma_{L-1} (L = tokens in the chunk):
//     E_r = exp(Gamma_r - Gamma_C) (>= 1),   F_r = exp(Gamma_C - Gamma_r) (<= 1)
//     Kt = k_r E_r,  Qt = scale q_r E_r,  Kb = k_r F_r                 (prep)
//     [A ; P] = [Kt ; Qt] Kb^T   (A_ri = sum_c k_rc k_ic e^{Gamma_rc - Gamma_ic})
//     M = strict_lower(diag(beta) A),  T' = (I + M)^-1 diag(beta)   (UT transform)
//     P = lower_incl(P)
//     U = T' V,  W' = T' Kt                                          (WY products)
//     St = Diag(exp(Gamma_C)) S                     (state decayed to chunk end)
//     delta = U - W' St,  O = Qt St + P delta,  S_next = St + Kb^T delta
// Unrolling the per-token rule inside the chunk gives (I + M) delta =
// diag(beta)(V - K~ S) with K~_r = k_r exp(Gamma_r) = Kt_r exp(Gamma_C), which
// is the triangular system above; O and S_next follow the same way.  Every
// exponent is taken relative to the chunk end, so all factors are finite as
// long as a channel's decay inside one chunk, -sum(g), stays below ~87.
//
// Precision: operands are rounded to tf32 (10-bit mantissa) and accumulated in
// fp32.  bf16 operands were measured (CPU emulation against the fp64 oracle)
// to exceed a 2e-2 x RMS max-error budget on the 8K-token workload; tf32 stays
// near 5e-3.  The state stays fp32 between chunks.
//
// Work decomposition: one CTA per (sequence, head, 32-column value slice); the
// value columns of S evolve independently, so four CTAs share a head and each
// recomputes the head-level chunk quantities (A, P, T', W').  Every MMA is
// M = 128 by stacking two 64-row operands:
//     [Kt ; Qt] x Kb^T      -> A (lanes 0-63), P (lanes 64-127)
//     [T' ; P]  x V         -> U (lanes 0-63; lanes 64-127 unused)
//     [T' ; P]  x Kt        -> W' (lanes 0-63; lanes 64-127 unused)
//     [-W' ; Qt] x St       -> -W' St (lanes 0-63), Qt St (lanes 64-127)
//     [T' ; P]  x delta     -> accumulated onto the previous: lanes 64-127 = O
//     Kb^T      x delta     -> accumulated onto St in TMEM: S_next
// Block: 256 threads (8 warps); thread 0 issues TMA and MMA.  A warp may only
// touch tensor-memory lanes 32*(warp%4) .. +31.
#include "kda_common.cuh"
#include "kda_launch.h"
#include "sm100.cuh"

#include <mutex>

namespace kda {
namespace {

constexpr int kC = 64;          // tokens per chunk
constexpr int kNV = 32;         // value columns per CTA
constexpr int kSplit = kD / kNV;
constexpr int kThreads = 256;

// Shared memory (byte offsets from a 1024-aligned base).  All MMA operand
// tiles use 128-byte rows with the 128-byte swizzle (see sm100.cuh).
constexpr uint32_t OFF_XQ = 0;        // 64 KB: 4 K-blocks (channels 32kb..) x 128 rows:
                                      //   rows 0-63 Kt (later -W'), rows 64-127 Qt
constexpr uint32_t OFF_KB = 65536;    // 32 KB: 4 K-blocks x 64 rows: Kb
constexpr uint32_t OFF_TP = 98304;    // 32 KB: 2 K-blocks (tokens 32kb..) x 128 rows:
                                      //   rows 0-63 T (fp32 while solving, then T'), rows 64-127 P
constexpr uint32_t OFF_SB = 131072;   // 16 KB: 128 rows (key channel) x 32 value cols: St;
                                      //   during the triangular solve: M (64 x 64 fp32)
constexpr uint32_t OFF_DL = 147456;   // 8 KB: 64 rows (token) x 32 value cols: delta;
                                      //   during prep: Gamma exchange; during the solve: temps
constexpr uint32_t OFF_VB = 155648;   // 8 KB: 64 rows (token) x 32 value cols: V slice
constexpr uint32_t OFF_RQ = 163840;   // 16 KB: raw q [64][128] bf16 (TMA destination)
constexpr uint32_t OFF_RK = 180224;   // 16 KB: raw k
constexpr uint32_t OFF_MISC = 196608; // beta[64], exp(Gamma_C)[128], barriers, TMEM address
constexpr uint32_t SMEM_BYTES = OFF_MISC + 1024 + 1024;   // + alignment slack

constexpr uint32_t KB_XQ = 16384;     // K-block strides
constexpr uint32_t KB_KB = 8192;
constexpr uint32_t KB_TP = 16384;

// Tensor-memory columns (fp32 accumulators, 128 lanes each).
constexpr uint32_t TM_AP = 0;     // 64 cols: A | P
constexpr uint32_t TM_U = 64;     // 32 cols: U
constexpr uint32_t TM_X = 96;     // 32 cols: -W'St | QtSt (+P delta = O)
constexpr uint32_t TM_W = 128;    // 128 cols: W'
constexpr uint32_t TM_S = 256;    // 32 cols: state slice (key rows x 32 value cols)
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t ID_AP = idesc_tf32(128, 64, false, false);
constexpr uint32_t ID_U = idesc_tf32(128, 32, false, true);
constexpr uint32_t ID_W = idesc_tf32(128, 128, false, true);
constexpr uint32_t ID_X = idesc_tf32(128, 32, false, true);
constexpr uint32_t ID_S = idesc_tf32(128, 32, true, true);

// fp32 scratch addressing inside the swizzled regions -----------------------
// M (64 x 64 fp32) in the St region: 16 float4 chunks per row, chunk position
// XOR-ed with the row so column-wise accesses of 32 rows hit distinct banks.
__device__ __forceinline__ float* M_at(uint8_t* smem, int r, int i) {
    return reinterpret_cast<float*>(smem + OFF_SB) + r * 64 + ((((i >> 2) ^ (r & 15))) << 2) + (i & 3);
}
// T / T' (rows 0-63 of the [T' ; P] operand, K-major, tokens along K).
__device__ __forceinline__ float* T_at(uint8_t* smem, int r, int i) {
    return reinterpret_cast<float*>(smem + OFF_TP + (i >> 5) * KB_TP + sw128_off(r, (i & 31) >> 2)) + (i & 3);
}

__device__ __forceinline__ void st_tf32x4(uint8_t* smem, uint32_t off, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(smem + off) = make_float4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}

// Store 32 consecutive fp32 values (one thread's TMEM row) as tf32 into the
// 8 chunks of swizzled row `row` of a region at byte offset `base`.
__device__ __forceinline__ void st_row32(uint8_t* smem, uint32_t base, int row, const float (&v)[32],
                                         float sign = 1.f) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
        st_tf32x4(smem, base + sw128_off(row, j), sign * v[4 * j], sign * v[4 * j + 1],
                  sign * v[4 * j + 2], sign * v[4 * j + 3]);
}

__device__ __forceinline__ uint32_t tm_lane(uint32_t tmem, int quarter, uint32_t col) {
    return tmem + (static_cast<uint32_t>(32 * quarter) << 16) + col;
}

__global__ void __launch_bounds__(kThreads, 1)
kda_chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __nv_bfloat16* __restrict__ v, const float* __restrict__ g,
                 const float* __restrict__ beta, const int32_t* __restrict__ cu_seqlens,
                 int64_t total_T, int H, float scale, int l2norm, const float* s0, float* sT,
                 float* __restrict__ o, uint32_t* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    float* beta_s = reinterpret_cast<float*>(smem + OFF_MISC);     // 64
    float* dc_s = beta_s + 64;                                      // 128: exp(Gamma_C)
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(smem + OFF_MISC + 768);
    uint64_t* bar_mma = bar_load + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 1);

    const int bid = blockIdx.x;
    const int slice = bid % kSplit;
    const int h = (bid / kSplit) % H;
    const int n = bid / (kSplit * H);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;

    const int64_t bos = cu_seqlens[n], eos = cu_seqlens[n + 1];
    if (bos < 0 || eos < bos || eos > total_T) {
        if (tid == 0 && slice == 0 && h == 0) set_error(err, 1u);
        return;   // inconsistent cu_seqlens: this sequence is skipped
    }
    const int64_t len = eos - bos;
    const int nchunks = static_cast<int>((len + kC - 1) / kC);

    if (warp == 0) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const size_t state_off = ((size_t)n * H + h) * kD * kD;

    // initial state slice -> TMEM (key row = lane, 32 value columns)
    if (warp < 4) {
        float r[32];
        const int row = 32 * warp + lane;
        if (s0) {
            const float4* src = reinterpret_cast<const float4*>(s0 + state_off + (size_t)row * kD + slice * kNV);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 x = src[j];
                r[4 * j] = x.x; r[4 * j + 1] = x.y; r[4 * j + 2] = x.z; r[4 * j + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = 0.f;
        }
        tmem_st32(tm_lane(tmem, warp, TM_S), r);
        tmem_wait_st();
    }

    // register-staged inputs of the next chunk: g (8 rows x 4 channels),
    // the thread's 8 values of the V slice, and beta
    float greg[8][4];
    uint4 vreg;
    float breg;
    auto prefetch = [&](int64_t t0, int L) {
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int r = 8 * warp + m;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < L) x = __ldg(reinterpret_cast<const float4*>(g + ((size_t)(t0 + r) * H + h) * kD + 4 * lane));
            greg[m][0] = x.x; greg[m][1] = x.y; greg[m][2] = x.z; greg[m][3] = x.w;
        }
        const int vr = tid >> 2;
        vreg = make_uint4(0u, 0u, 0u, 0u);
        if (vr < L)
            vreg = __ldg(reinterpret_cast<const uint4*>(v + ((size_t)(t0 + vr) * H + h) * kD + slice * kNV + 8 * (tid & 3)));
        breg = 0.f;
        if (tid < L) breg = __ldg(beta + (size_t)(t0 + tid) * H + h);
    };
    auto issue_load = [&](int64_t t0) {
        mbar_arrive_expect_tx(bar_load, 2u * kC * kD * 2u);
        tma_load_3d(smem + OFF_RQ, &tm_q, bar_load, 0, h, static_cast<int32_t>(t0));
        tma_load_3d(smem + OFF_RK, &tm_k, bar_load, 0, h, static_cast<int32_t>(t0));
    };

    bool ok = true;
    uint32_t mma_phase = 0;
    bool load_pending = false, mma_pending = false;
    uint32_t load_parity = 0;
    if (nchunks > 0) {
        if (tid == 0) issue_load(bos);
        load_pending = true;
        prefetch(bos, static_cast<int>((len < kC ? len : (int64_t)kC)));
    }
    tc_fence_before();
    __syncthreads();

    for (int c = 0; c < nchunks; ++c) {
        const int64_t t0 = bos + (int64_t)c * kC;
        const int L = static_cast<int>((eos - t0 < kC ? eos - t0 : (int64_t)kC));

        ok = !__syncthreads_or(!mbar_wait_bounded(bar_load, c & 1));
        if (!ok) break;
        load_pending = false;

        // ---------------------------------------------------------- prep
        {
            float* xch = reinterpret_cast<float*>(smem + OFF_DL);   // [8 warps][128]
            float G[8][4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                float run = 0.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    run = fmaf(greg[m][x], kLog2e, run);
                    G[m][x] = run;
                }
                xch[warp * 128 + 4 * lane + x] = run;
            }
            __syncthreads();
            float off[4] = {0.f, 0.f, 0.f, 0.f}, GC[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                const float4 t = *reinterpret_cast<const float4*>(xch + w * 128 + 4 * lane);
                if (w < warp) { off[0] += t.x; off[1] += t.y; off[2] += t.z; off[3] += t.w; }
                GC[0] += t.x; GC[1] += t.y; GC[2] += t.z; GC[3] += t.w;
            }
            if (warp == 0) {
#pragma unroll
                for (int x = 0; x < 4; ++x) dc_s[4 * lane + x] = ex2(GC[x]);
            }
            if (tid < kC) beta_s[tid] = breg;

            const __nv_bfloat16* rq = reinterpret_cast<const __nv_bfloat16*>(smem + OFF_RQ);
            const __nv_bfloat16* rk = reinterpret_cast<const __nv_bfloat16*>(smem + OFF_RK);
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int r = 8 * warp + m;
                float qv[4], kv[4];
                load4(rq + r * kD + 4 * lane, qv);
                load4(rk + r * kD + 4 * lane, kv);
                if (r >= L) {
#pragma unroll
                    for (int x = 0; x < 4; ++x) { qv[x] = 0.f; kv[x] = 0.f; }
                }
                float nq = 1.f, nk = 1.f;
                if (l2norm) {
                    float sq = 0.f, sk = 0.f;
#pragma unroll
                    for (int x = 0; x < 4; ++x) { sq = fmaf(qv[x], qv[x], sq); sk = fmaf(kv[x], kv[x], sk); }
                    nq = rsqrtf(warp_sum(sq) + kNormEps);
                    nk = rsqrtf(warp_sum(sk) + kNormEps);
                }
                nq *= scale;
                float kt[4], qt[4], kb[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float gr = G[m][x] + off[x];
                    const float e = ex2(fminf(gr - GC[x], 126.f));   // exp(Gamma_r - Gamma_C) >= 1
                    const float f = ex2(GC[x] - gr);                 // exp(Gamma_C - Gamma_r) <= 1
                    const float kn = kv[x] * nk;
                    kt[x] = kn * e;
                    kb[x] = kn * f;
                    qt[x] = qv[x] * nq * e;
                }
                const int kbi = lane >> 3, ch = lane & 7;
                st_tf32x4(smem, OFF_XQ + kbi * KB_XQ + sw128_off(r, ch), kt[0], kt[1], kt[2], kt[3]);
                st_tf32x4(smem, OFF_XQ + kbi * KB_XQ + sw128_off(64 + r, ch), qt[0], qt[1], qt[2], qt[3]);
                st_tf32x4(smem, OFF_KB + kbi * KB_KB + sw128_off(r, ch), kb[0], kb[1], kb[2], kb[3]);
            }
            {   // V slice: token tid/4, value columns 8*(tid%4) .. +7 (exact bf16 -> fp32)
                const int r = tid >> 2, cp = 2 * (tid & 3);
                const uint32_t w4[4] = {vreg.x, vreg.y, vreg.z, vreg.w};
                float f[8];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    f[2 * x] = __uint_as_float(w4[x] << 16);
                    f[2 * x + 1] = __uint_as_float(w4[x] & 0xFFFF0000u);
                }
                *reinterpret_cast<float4*>(smem + OFF_VB + sw128_off(r, cp)) = make_float4(f[0], f[1], f[2], f[3]);
                *reinterpret_cast<float4*>(smem + OFF_VB + sw128_off(r, cp + 1)) = make_float4(f[4], f[5], f[6], f[7]);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---------------------------------------- next loads, A/P product
        if (tid == 0) {
            if (c + 1 < nchunks) issue_load(t0 + kC);
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 16; ++s) {
                const uint64_t a = sdesc_sw128(sb + OFF_XQ + (s >> 2) * KB_XQ + (s & 3) * 32, 16, 1024);
                const uint64_t b = sdesc_sw128(sb + OFF_KB + (s >> 2) * KB_KB + (s & 3) * 32, 16, 1024);
                mma_tf32_ss(tmem + TM_AP, a, b, ID_AP, s > 0);
            }
            mma_commit(bar_mma);
        }
        load_pending = (c + 1 < nchunks);
        load_parity = (c + 1) & 1;
        mma_pending = true;
        if (c + 1 < nchunks) prefetch(t0 + kC, static_cast<int>((eos - t0 - kC < kC ? eos - t0 - kC : (int64_t)kC)));
        ok = !__syncthreads_or(!mbar_wait_bounded(bar_mma, mma_phase));
        if (!ok) break;
        mma_phase ^= 1;
        mma_pending = false;
        tc_fence_after();

        // ------------------------------- A -> M (fp32), P -> tf32 operand
        {
            float acc[32];
            tmem_ld32(tm_lane(tmem, quarter, TM_AP + 32 * half), acc);
            tmem_wait_ld();
            if (quarter < 2) {
                const int r = 32 * quarter + lane;
                const float br = beta_s[r];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float4 x;
                    const int i0 = 32 * half + 4 * j;
                    x.x = (i0 + 0 < r) ? br * acc[4 * j + 0] : 0.f;
                    x.y = (i0 + 1 < r) ? br * acc[4 * j + 1] : 0.f;
                    x.z = (i0 + 2 < r) ? br * acc[4 * j + 2] : 0.f;
                    x.w = (i0 + 3 < r) ? br * acc[4 * j + 3] : 0.f;
                    *reinterpret_cast<float4*>(M_at(smem, r, i0)) = x;
                }
            } else {
                const int r = 32 * quarter + lane - 64;
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    if (32 * half + e > r) acc[e] = 0.f;
                st_row32(smem, OFF_TP + half * KB_TP, 64 + r, acc);
            }
        }
        tc_fence_before();
        __syncthreads();

        // ------------------------- T = (I + M)^-1 by 16-blocks, then T' = T diag(beta)
        {
            float* tmpY = reinterpret_cast<float*>(smem + OFF_DL);
            if (tid < 64) {   // diagonal 16 x 16 blocks: column j of block b by substitution
                const int b = tid >> 4, j = tid & 15;
                float xv[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float s = (r == j) ? 1.f : 0.f;
#pragma unroll
                    for (int i = 0; i < r; ++i) s = fmaf(-*M_at(smem, 16 * b + r, 16 * b + i), xv[i], s);
                    xv[r] = s;
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) *T_at(smem, 16 * b + r, 16 * b + j) = xv[r];
            } else {          // zero the six blocks above the diagonal
                for (int e = tid - 64; e < 6 * 256; e += kThreads - 64) {
                    // block index 0..5 -> (row block, col block) = (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
                    const int blk = e >> 8, w = e & 255, rr = w >> 4, jj = w & 15;
                    const int rb = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
                    const int cb = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
                    *T_at(smem, 16 * rb + rr, 16 * cb + jj) = 0.f;
                }
            }
            __syncthreads();
            {   // 16 -> 32: T_ab = -T_aa M_ab T_bb for (a, b) = (1, 0), (3, 2)
                const int p = tid >> 7, rr = (tid & 127) >> 3, j0 = (tid & 7) * 2;
                const int a = 2 * p + 1, b = 2 * p;
                float y0 = 0.f, y1 = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float mv = *M_at(smem, 16 * a + rr, 16 * b + i);
                    y0 = fmaf(mv, *T_at(smem, 16 * b + i, 16 * b + j0), y0);
                    y1 = fmaf(mv, *T_at(smem, 16 * b + i, 16 * b + j0 + 1), y1);
                }
                tmpY[p * 256 + rr * 16 + j0] = y0;
                tmpY[p * 256 + rr * 16 + j0 + 1] = y1;
                __syncthreads();
                float z0 = 0.f, z1 = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float tv = *T_at(smem, 16 * a + rr, 16 * a + i);
                    z0 = fmaf(tv, tmpY[p * 256 + i * 16 + j0], z0);
                    z1 = fmaf(tv, tmpY[p * 256 + i * 16 + j0 + 1], z1);
                }
                *T_at(smem, 16 * a + rr, 16 * b + j0) = -z0;
                *T_at(smem, 16 * a + rr, 16 * b + j0 + 1) = -z1;
            }
            __syncthreads();
            {   // 32 -> 64: T_hl = -T_hh M_hl T_ll with 32 x 32 blocks
                const int rr = tid >> 3, j0 = (tid & 7) * 4;
                float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
                for (int i = 0; i < 32; ++i) {
                    const float mv = *M_at(smem, 32 + rr, i);
                    const float4 t4 = *reinterpret_cast<const float4*>(T_at(smem, i, j0));
                    y[0] = fmaf(mv, t4.x, y[0]); y[1] = fmaf(mv, t4.y, y[1]);
                    y[2] = fmaf(mv, t4.z, y[2]); y[3] = fmaf(mv, t4.w, y[3]);
                }
                *reinterpret_cast<float4*>(tmpY + rr * 32 + j0) = make_float4(y[0], y[1], y[2], y[3]);
                __syncthreads();
                float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
                for (int i = 0; i < 32; ++i) {
                    const float tv = *T_at(smem, 32 + rr, 32 + i);
                    const float4 y4 = *reinterpret_cast<const float4*>(tmpY + i * 32 + j0);
                    z[0] = fmaf(tv, y4.x, z[0]); z[1] = fmaf(tv, y4.y, z[1]);
                    z[2] = fmaf(tv, y4.z, z[2]); z[3] = fmaf(tv, y4.w, z[3]);
                }
                *reinterpret_cast<float4*>(T_at(smem, 32 + rr, j0)) = make_float4(-z[0], -z[1], -z[2], -z[3]);
            }
            __syncthreads();
            {   // T' = T diag(beta), rounded to tf32
                const int r = tid >> 2;
#pragma unroll
                for (int qd = 0; qd < 4; ++qd) {
                    const int i0 = 16 * (tid & 3) + 4 * qd;
                    float4* p4 = reinterpret_cast<float4*>(T_at(smem, r, i0));
                    const float4 t4 = *p4;
                    *p4 = make_float4(to_tf32(t4.x * beta_s[i0]), to_tf32(t4.y * beta_s[i0 + 1]),
                                      to_tf32(t4.z * beta_s[i0 + 2]), to_tf32(t4.w * beta_s[i0 + 3]));
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ------------------------------------- U = T' V, W' = T' Kt
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint64_t a = sdesc_sw128(sb + OFF_TP + (s >> 2) * KB_TP + (s & 3) * 32, 16, 1024);
                const uint64_t bv = sdesc_sw128(sb + OFF_VB + s * 1024, 8192, 1024);
                const uint64_t bk = sdesc_sw128(sb + OFF_XQ + s * 1024, KB_XQ, 1024);
                mma_tf32_ss(tmem + TM_U, a, bv, ID_U, s > 0);
                mma_tf32_ss(tmem + TM_W, a, bk, ID_W, s > 0);
            }
            mma_commit(bar_mma);
        }
        mma_pending = true;
        // meanwhile: decay the state to the chunk end, St = Diag(exp(Gamma_C)) S,
        // in TMEM (fp32) and as the tf32 operand
        if (warp < 4) {
            float acc[32];
            tc_fence_after();
            tmem_ld32(tm_lane(tmem, warp, TM_S), acc);
            tmem_wait_ld();
            const int row = 32 * warp + lane;
            const float dcr = dc_s[row];
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[e] *= dcr;
            tmem_st32(tm_lane(tmem, warp, TM_S), acc);
            st_row32(smem, OFF_SB, row, acc);
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        ok = !__syncthreads_or(!mbar_wait_bounded(bar_mma, mma_phase));
        if (!ok) break;
        mma_phase ^= 1;
        mma_pending = false;
        tc_fence_after();

        // ------------------------------------- -W' -> rows 0-63 of the XQ stack
        if (quarter < 2) {
            const int r = 32 * quarter + lane;
#pragma unroll
            for (int m2 = 0; m2 < 2; ++m2) {
                float acc[32];
                tmem_ld32(tm_lane(tmem, quarter, TM_W + 64 * half + 32 * m2), acc);
                tmem_wait_ld();
                st_row32(smem, OFF_XQ + (2 * half + m2) * KB_XQ, r, acc, -1.f);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ------------------------------------- [-W' ; Qt] St
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 16; ++s) {
                const uint64_t a = sdesc_sw128(sb + OFF_XQ + (s >> 2) * KB_XQ + (s & 3) * 32, 16, 1024);
                const uint64_t b = sdesc_sw128(sb + OFF_SB + s * 1024, 8192, 1024);
                mma_tf32_ss(tmem + TM_X, a, b, ID_X, s > 0);
            }
            mma_commit(bar_mma);
        }
        mma_pending = true;
        ok = !__syncthreads_or(!mbar_wait_bounded(bar_mma, mma_phase));
        if (!ok) break;
        mma_phase ^= 1;
        mma_pending = false;
        tc_fence_after();

        // ------------------------------------- delta = U - W' St (token rows 0-63)
        if (warp < 2) {
            float x[32], u[32];
            tmem_ld32(tm_lane(tmem, warp, TM_X), x);
            tmem_ld32(tm_lane(tmem, warp, TM_U), u);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] += u[e];
            st_row32(smem, OFF_DL, 32 * warp + lane, x);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ------------------------------------- O += P delta, S = St + Kb^T delta
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint64_t a = sdesc_sw128(sb + OFF_TP + (s >> 2) * KB_TP + (s & 3) * 32, 16, 1024);
                const uint64_t bd = sdesc_sw128(sb + OFF_DL + s * 1024, 8192, 1024);
                const uint64_t ak = sdesc_sw128(sb + OFF_KB + s * 1024, KB_KB, 1024);
                mma_tf32_ss(tmem + TM_X, a, bd, ID_X, 1);
                mma_tf32_ss(tmem + TM_S, ak, bd, ID_S, 1);
            }
            mma_commit(bar_mma);
        }
        mma_pending = true;
        ok = !__syncthreads_or(!mbar_wait_bounded(bar_mma, mma_phase));
        if (!ok) break;
        mma_phase ^= 1;
        mma_pending = false;
        tc_fence_after();

        // ------------------------------------- O (token rows, lanes 64-127) -> global
        if (warp == 2 || warp == 3) {
            float acc[32];
            tmem_ld32(tm_lane(tmem, warp, TM_X), acc);
            tmem_wait_ld();
            const int r = 32 * warp + lane - 64;
            if (r < L) {
                float4* dst = reinterpret_cast<float4*>(o + ((size_t)(t0 + r) * H + h) * kD + slice * kNV);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    dst[j] = make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
            }
        }
        tc_fence_before();
        __syncthreads();
    }

    if (ok) {
        if (sT && warp < 4) {
            float acc[32];
            tc_fence_after();
            tmem_ld32(tm_lane(tmem, warp, TM_S), acc);
            tmem_wait_ld();
            float4* dst = reinterpret_cast<float4*>(sT + state_off + (size_t)(32 * warp + lane) * kD + slice * kNV);
#pragma unroll
            for (int j = 0; j < 8; ++j) dst[j] = make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
        }
    } else {
        // a bounded wait gave up: report, give outstanding copies and MMAs a
        // last bounded chance to land, then release tensor memory
        if (tid == 0) {
            set_error(err, 2u);
            if (load_pending) mbar_wait_bounded(bar_load, load_parity, 1u << 16);
            if (mma_pending) mbar_wait_bounded(bar_mma, mma_phase, 1u << 16);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [total_T, H, 128] bf16 viewed as a 3-D tensor (channel, head, token); one
// box is 64 tokens x 128 channels of one head, no swizzle.
bool make_qk_map(CUtensorMap* map, const void* base, int64_t total_T, int H) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(total_T)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD) * 2, static_cast<cuuint64_t>(H) * kD * 2};
    cuuint32_t box[3] = {kD, 1, kC};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunk(const PrefillArgs& a, cudaStream_t stream) {
    if (a.N == 0 || a.H == 0) return cudaSuccess;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(kda_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(SMEM_BYTES));
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap mq, mk;
    // a zero-token batch still needs valid maps; point them at a 1-token extent
    const int64_t extent = a.total_T > 0 ? a.total_T : 1;
    if (!make_qk_map(&mq, a.q, extent, a.H) || !make_qk_map(&mk, a.k, extent, a.H))
        return cudaErrorInvalidValue;
    const long long blocks = (long long)a.N * a.H * kSplit;
    kda_chunk_kernel<<<static_cast<unsigned>(blocks), kThreads, SMEM_BYTES, stream>>>(
        mq, mk, static_cast<const __nv_bfloat16*>(a.v), a.g, a.beta, a.cu_seqlens, a.total_T, a.H, a.scale,
        a.l2norm ? 1 : 0, a.initial_state, a.final_state, a.o, a.err);
    return cudaGetLastError();
}

}  // namespace kda
