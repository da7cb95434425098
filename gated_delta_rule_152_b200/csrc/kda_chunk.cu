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
//     Kt = k_r E_r,  Qt = scale q_r E_r,  Kb = k_r F_r                  (prep)
//     St = Diag(exp(Gamma_C)) S                     (state decayed to chunk end)
//     [A ; P] = [Kt ; Qt] Kb^T   (A_ri = sum_c k_rc k_ic e^{Gamma_rc - Gamma_ic})
//     [Y ; Z] = [Kt ; Qt] St     (Y_r = k_r^T Diag(e^{Gamma_r}) S, Z_r likewise for q)
//     M = strict_lower(diag(beta) A),  T' = (I + M)^-1 diag(beta)   (UT transform)
//     delta = T' (V - Y),   O = Z + lower_incl(P) delta,   S_next = St + Kb^T delta
// Unrolling the per-token rule inside the chunk gives the triangular system
// (I + M) delta = diag(beta) (V - Y) for the rank-one corrections delta_r,
// from which the outputs and the end state follow.  Every exponent is taken
// relative to the chunk end, so the factors stay inside the fp32 range while a
// channel's decay inside one chunk, -sum(g), stays below 100 log2 units (about
// 69 nats; level 0 of kda_tile.cuh).  A chunk that decays more in some
// channel -- the page lets every channel decay at its own data-dependent
// rate, so nothing bounds it -- sends its (sequence, head, slice) to the
// token-by-token recurrence (serial_slice, kda_serial.cuh), which restarts from
// the initial state; the two-pass kernels handle such chunks in place.
//
// Precision: operands are rounded to tf32 (10-bit mantissa) and accumulated in
// fp32.  bf16 operands were measured (CPU emulation against the fp64 oracle)
// to exceed a 2e-2 x RMS max-error budget on the 8K-token workload; tf32 stays
// near 5e-3.  The state stays fp32 between chunks (in tensor memory).
//
// Work decomposition: one CTA per (sequence, head, 32-column value slice); the
// value columns of S evolve independently, so four CTAs share a head and each
// recomputes the head-level chunk quantities (A, P, T').  Every MMA is
// M = 128 (two 64-row operands stacked) with both operands K-major in shared
// memory:
//     [Kt ; Qt] x [Kb^T | St] -> A | Y (lanes 0-63), P | Z (lanes 64-127), N = 96
//     [T' ; P]  x (V - Y)   -> delta (lanes 0-63; lanes 64-127 unused)
//     [T' ; P]  x delta    -> accumulated onto [Y ; Z]: lanes 64-127 = O
//     Kb^T      x delta    -> accumulated onto St in TMEM: S_next
// Block: 256 threads (8 warps); thread 0 issues TMA and MMA.  A warp may only
// touch tensor-memory lanes 32*(warp%4) .. +31.
#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_serial.cuh"
#include "kda_tile.cuh"
#include "sm100.cuh"

#include <mutex>

namespace kda {
namespace {

constexpr int kC = 64;          // tokens per chunk
constexpr int kNV = 32;         // value columns per CTA
constexpr int kSplit = kD / kNV;
constexpr int kThreads = 256;

// Shared memory (byte offsets from a 1024-aligned base).  Every MMA operand
// is K-major with 128-byte rows (32 tf32 elements of K) and the 128-byte
// swizzle (sm100.cuh); further K elements live in further "K-blocks".
constexpr uint32_t OFF_XQ = 0;         // 64 KB: [Kt ; Qt], 128 rows (token, token) x 128 channels
                                       //   = 4 K-blocks x 16 KB.  After the first MMA pair it is
                                       //   dead and holds the triangular solve's scratch.
constexpr uint32_t OFF_KS = 65536;     // 48 KB: [Kb ; St^T], 96 rows x 128 channels = 4 K-blocks x 12 KB:
                                       //   rows 0-63 Kb (token), rows 64-95 St^T (value column).
                                       //   Also the TMA destination of the next chunk's raw q, k.
constexpr uint32_t OFF_KBT = 114688;   // 32 KB: Kb^T, 128 rows (channel) x 64 tokens = 2 K-blocks x 16 KB
constexpr uint32_t OFF_TP = 147456;    // 32 KB: [T' ; P], 128 rows x 64 tokens = 2 K-blocks x 16 KB
constexpr uint32_t OFF_VT = 180224;    // 8 KB: V^T, then (V - Y)^T: 32 rows x 64 tokens = 2 x 4 KB
constexpr uint32_t OFF_YT = 188416;    // 8 KB: delta^T
constexpr uint32_t OFF_MISC = 196608;  // beta[64], exp(Gamma_C)[128], Gamma exchange [8][128],
                                       //   barriers, TMEM address
constexpr uint32_t SMEM_BYTES = OFF_MISC + 6144 + 1024;   // + alignment slack

constexpr uint32_t KB_XQ = 16384;      // K-block strides
constexpr uint32_t KB_KS = 12288;
constexpr uint32_t KB_KBT = 16384;
constexpr uint32_t KB_TP = 16384;
constexpr uint32_t KB_VT = 4096;

// Scratch of the triangular solve inside the dead XQ region (kda_tile.cuh).
constexpr uint32_t OFF_M = OFF_XQ;                         // M, 64 x kLd
constexpr uint32_t OFF_T = OFF_M + 64 * kLd * 4;           // T, 64 x kLd
constexpr uint32_t OFF_Y1 = OFF_T + 64 * kLd * 4;          // 2 x 16 x kLd1
constexpr uint32_t OFF_Y2 = OFF_Y1 + 2 * 16 * kLd1 * 4;    // 32 x kLd2
static_assert(OFF_Y2 + 32 * kLd2 * 4 <= OFF_XQ + 65536, "solve scratch exceeds the XQ region");

// Tensor-memory columns (fp32 accumulators, 128 lanes each).
constexpr uint32_t TM_AP = 0;     // 64 cols: A | P
constexpr uint32_t TM_X = 64;     // 32 cols: Y | Z, then Z + P delta = O in lanes 64-127
constexpr uint32_t TM_U = 96;     // 32 cols: T'V, then delta in lanes 0-63
constexpr uint32_t TM_S = 128;    // 32 cols: state slice (key rows x 32 value cols)
constexpr uint32_t TM_COLS = 256;

constexpr uint32_t ID_N96 = idesc_tf32(128, 96, false, false);
constexpr uint32_t ID_N32 = idesc_tf32(128, 32, false, false);

__global__ void __launch_bounds__(kThreads, 1)
kda_chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                 const __nv_bfloat16* __restrict__ v, const float* __restrict__ g,
                 const float* __restrict__ beta, const int32_t* __restrict__ cu_seqlens,
                 int64_t total_T, int H, float scale, int l2norm, int scalar_g, const float* s0,
                 float* sT, float* __restrict__ o, uint32_t* err, const int32_t* __restrict__ slots,
                 int num_slots) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    float* beta_s = reinterpret_cast<float*>(smem + OFF_MISC);            // 64
    float* dc_s = beta_s + 64;                                             // 128: exp(Gamma_C)
    float* xch = reinterpret_cast<float*>(smem + OFF_MISC + 1024);         // [8 warps][128]
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(smem + OFF_MISC + 5120);
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
    // state index of this sequence: n, or its slot in a state pool
    const int64_t sidx = slots ? static_cast<int64_t>(slots[n]) : static_cast<int64_t>(n);
    if (slots && (sidx < 0 || sidx >= num_slots)) {
        if (tid == 0 && slice == 0 && h == 0) set_error(err, 4u);
        return;   // slot out of range: this sequence is skipped
    }

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
    const size_t state_off = ((size_t)sidx * H + h) * kD * kD;

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

    // Register-staged inputs of the next chunk: g (8 rows x 4 channels), the
    // thread's 8 values of the V slice, and beta.
    float greg[8][4];
    uint4 vreg;
    float breg;
    auto prefetch = [&](int64_t t0, int L) {
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int r = 8 * warp + m;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < L) {
                if (scalar_g) {   // one decay per (token, head), shared by all channels
                    const float gs = __ldg(g + (size_t)(t0 + r) * H + h);
                    x = make_float4(gs, gs, gs, gs);
                } else {
                    x = __ldg(reinterpret_cast<const float4*>(g + ((size_t)(t0 + r) * H + h) * kD + 4 * lane));
                }
            }
            greg[m][0] = x.x; greg[m][1] = x.y; greg[m][2] = x.z; greg[m][3] = x.w;
        }
        const int vr = tid >> 2;
        vreg = make_uint4(0u, 0u, 0u, 0u);
        if (vr < L)
            vreg = __ldg(reinterpret_cast<const uint4*>(v + ((size_t)(t0 + vr) * H + h) * kD + slice * kNV + 8 * (tid & 3)));
        breg = 0.f;
        if (tid < L) breg = __ldg(beta + (size_t)(t0 + tid) * H + h);
    };
    // raw q and k tiles (64 tokens x 128 channels, bf16) into the [Kb ; St^T] region
    auto issue_load = [&](int64_t t0) {
        mbar_arrive_expect_tx(bar_load, 2u * kC * kD * 2u);
        tma_load_3d(smem + OFF_KS, &tm_q, bar_load, 0, h, static_cast<int32_t>(t0));
        tma_load_3d(smem + OFF_KS + kC * kD * 2, &tm_k, bar_load, 0, h, static_cast<int32_t>(t0));
    };

    // Prep of one chunk (state independent): Gamma, L2 norms, the tf32 tiles
    // Kt, Qt (XQ), Kb (rows 0-63 of KS) and V^T, plus beta and exp(Gamma_C).
    // Returns the chunk's Gram level (kda_tile.cuh); this kernel's single
    // reference point per chunk serves level 0 only.  Contains one block
    // barrier; every thread must call it.
    auto prep = [&](int L) -> int {
        float4 gc;
        const int level = prep_chunk_rows(
            smem + OFF_KS, smem + OFF_KS + kC * kD * 2, greg, xch, L, scale, l2norm != 0,
            [&](const ChunkChannels& cc, int) { gc = cc.rho[3]; },
            [&](int r, int kbi, int ch, float4 qn, float4 kn, float4 gr) {
            // a = Gamma_r - Gamma_C >= 0 (the decay is cumulative, g <= 0): E = 2^a >= 1, F = 2^-a <= 1
            const float4 a = sub4(gr, gc);
            const float4 E = ex2x4(make_float4(fminf(a.x, 126.f), fminf(a.y, 126.f), fminf(a.z, 126.f), fminf(a.w, 126.f)));
            const float4 F = ex2x4(make_float4(-a.x, -a.y, -a.z, -a.w));
            const float4 kt = mul4(kn, E), qt = mul4(qn, E), kb = mul4(kn, F);
            st_tf32x4(smem, OFF_XQ + kbi * KB_XQ + sw128_off(r, ch), kt.x, kt.y, kt.z, kt.w);
            st_tf32x4(smem, OFF_XQ + kbi * KB_XQ + sw128_off(64 + r, ch), qt.x, qt.y, qt.z, qt.w);
            st_tf32x4(smem, OFF_KS + kbi * KB_KS + sw128_off(r, ch), kb.x, kb.y, kb.z, kb.w);
        });
        if (warp == 0) *reinterpret_cast<float4*>(dc_s + 4 * lane) = ex2x4(gc);
        if (tid < kC) beta_s[tid] = breg;
        {   // V^T: token tid/4, value columns 8*(tid%4) .. +7 (exact bf16 -> fp32)
            const int r = tid >> 2, j0 = 8 * (tid & 3);
            const uint32_t w4[4] = {vreg.x, vreg.y, vreg.z, vreg.w};
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                *K_at(smem, OFF_VT, KB_VT, j0 + 2 * x, r) = __uint_as_float(w4[x] << 16);
                *K_at(smem, OFF_VT, KB_VT, j0 + 2 * x + 1, r) = __uint_as_float(w4[x] & 0xFFFF0000u);
            }
        }
        return level;
    };

    bool ok = true;
    uint32_t mma_phase = 0, load_parity = 0;
    bool load_pending = false, mma_pending = false;
    auto wait_mma = [&]() -> bool {
        const bool good = !__syncthreads_or(!mbar_wait_bounded(bar_mma, mma_phase));
        if (good) {
            mma_phase ^= 1;
            mma_pending = false;
            tc_fence_after();
        }
        return good;
    };

    // level of the chunk prepared last: a chunk whose decay is too strong for the
    // chunk-end reference point sends the whole (sequence, head, slice) to the
    // token-by-token recurrence instead (serial_slice, from the initial state)
    int lvl_next = 0;
    if (nchunks > 0) {   // prologue: stage and prep chunk 0
        if (tid == 0) issue_load(bos);
        load_pending = true;
        prefetch(bos, static_cast<int>(len < kC ? len : (int64_t)kC));
        ok = !__syncthreads_or(!mbar_wait_bounded(bar_load, 0));
        if (ok) {
            load_pending = false;
            lvl_next = prep(static_cast<int>(len < kC ? len : (int64_t)kC));
        }
    }

    bool serial = false;
    for (int c = 0; ok && c < nchunks; ++c) {
        if (lvl_next != 0) {   // nothing is in flight here: chunk c's load was consumed by its prep
            serial = true;
            break;
        }
        const int64_t t0 = bos + (int64_t)c * kC;
        const int L = static_cast<int>(eos - t0 < kC ? eos - t0 : (int64_t)kC);
        const bool has_next = c + 1 < nchunks;
        const int Ln = has_next ? static_cast<int>(eos - t0 - kC < kC ? eos - t0 - kC : (int64_t)kC) : 0;
        tc_fence_before();
        __syncthreads();   // prep(c) done; the previous chunk's TMEM reads done

        // ============== Kb^T, and the state decayed to the chunk end
        {   // Kb^T from Kb: thread = channel c, 4 consecutive tokens per 16-byte
            // store; all 32 loads are issued before the first store
            const int cch = tid & 127, tg = tid >> 7;
            float4 x[8];
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                const int i0 = 32 * tg + 4 * b;
                x[b].x = *K_at(smem, OFF_KS, KB_KS, i0 + 0, cch);
                x[b].y = *K_at(smem, OFF_KS, KB_KS, i0 + 1, cch);
                x[b].z = *K_at(smem, OFF_KS, KB_KS, i0 + 2, cch);
                x[b].w = *K_at(smem, OFF_KS, KB_KS, i0 + 3, cch);
            }
#pragma unroll
            for (int b = 0; b < 8; ++b)
                *reinterpret_cast<float4*>(K_at(smem, OFF_KBT, KB_KBT, cch, 32 * tg + 4 * b)) = x[b];
        }
        {   // St = Diag(exp(Gamma_C)) S in TMEM (fp32) and as St^T (tf32, rows 64-95 of KS);
            // the two warps of a TMEM lane quarter take 16 value columns each
            float acc[16];
            const int c0 = 16 * half;
            tc_fence_after();
            tmem_ld16(tm_lane(tmem, quarter, TM_S + c0), acc);
            tmem_wait_ld();
            const int row = 32 * quarter + lane;
            const float dcr = dc_s[row];
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[e] *= dcr;
            tmem_st16(tm_lane(tmem, quarter, TM_S + c0), acc);
#pragma unroll
            for (int e = 0; e < 16; ++e) *K_at(smem, OFF_KS, KB_KS, 64 + c0 + e, row) = to_tf32(acc[e]);
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ============== [Kt ; Qt] x [Kb ; St^T]^T -> [A | Y] (lanes 0-63), [P | Z] (64-127)
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dxq = tdesc(sb, OFF_XQ), dks = tdesc(sb, OFF_KS);
#pragma unroll
            for (int s = 0; s < 16; ++s)
                mma_tf32_ss(tmem + TM_AP, kstep(dxq, KB_XQ, s), kstep(dks, KB_KS, s), ID_N96, s > 0);
            mma_commit(bar_mma);
        }
        mma_pending = true;
        if (has_next) prefetch(t0 + kC, Ln);
        if (!(ok = wait_mma())) break;
        // XQ and KS are free now: stage the next chunk's q, k
        if (tid == 0 && has_next) issue_load(t0 + kC);
        load_pending = has_next;
        load_parity = (c + 1) & 1;

        // ============== A -> M (fp32), P -> tf32 operand
        {
            float acc[32];
            tmem_ld32(tm_lane(tmem, quarter, TM_AP + 32 * half), acc);
            tmem_wait_ld();
            if (quarter < 2) {
                const int r = 32 * quarter + lane;
                const float br = beta_s[r];
                float* mrow = reinterpret_cast<float*>(smem + OFF_M) + r * kLd + 32 * half;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float4 x;
                    const int i0 = 32 * half + 4 * j;
                    x.x = (i0 + 0 < r) ? br * acc[4 * j + 0] : 0.f;
                    x.y = (i0 + 1 < r) ? br * acc[4 * j + 1] : 0.f;
                    x.z = (i0 + 2 < r) ? br * acc[4 * j + 2] : 0.f;
                    x.w = (i0 + 3 < r) ? br * acc[4 * j + 3] : 0.f;
                    *reinterpret_cast<float4*>(mrow + 4 * j) = x;
                }
            } else {
                const int r = 32 * quarter + lane - 64;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int i0 = 32 * half + 4 * j;
                    st_tf32x4(smem, OFF_TP + half * KB_TP + sw128_off(64 + r, j),
                              (i0 + 0 <= r) ? acc[4 * j + 0] : 0.f, (i0 + 1 <= r) ? acc[4 * j + 1] : 0.f,
                              (i0 + 2 <= r) ? acc[4 * j + 2] : 0.f, (i0 + 3 <= r) ? acc[4 * j + 3] : 0.f);
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ============== T = (I + M)^-1 by 16-blocks, then T' = T diag(beta);
        // meanwhile V^T -> (V - Y)^T
        {
            float* Mf = reinterpret_cast<float*>(smem + OFF_M);
            float* Tf = reinterpret_cast<float*>(smem + OFF_T);
            float* Y1 = reinterpret_cast<float*>(smem + OFF_Y1);   // [2][16][kLd1]
            float* Y2 = reinterpret_cast<float*>(smem + OFF_Y2);   // [32][kLd2]
            ut_inverse64(Mf, Tf, Y1, Y2, tid, [&] {
                if (warp == 4 || warp == 5) {   // V^T -> (V - Y)^T for token rows 0-63
                    float y[32];
                    tc_fence_after();
                    tmem_ld32(tm_lane(tmem, quarter, TM_X), y);
                    tmem_wait_ld();
                    const int r = 32 * quarter + lane;
                    // all loads before all stores: the compiler cannot prove the
                    // 32 addresses distinct, so an interleaved read-modify-write
                    // would serialise on shared-memory latency
                    float vv[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) vv[e] = *K_at(smem, OFF_VT, KB_VT, e, r);
#pragma unroll
                    for (int e = 0; e < 32; ++e) *K_at(smem, OFF_VT, KB_VT, e, r) = to_tf32(vv[e] - y[e]);
                }
            });
            {   // T' = T diag(beta) on and below the diagonal, zero above; tf32 operand
                const int r = tid >> 2;
                float4 t4[4], b4[4];
#pragma unroll
                for (int qd = 0; qd < 4; ++qd) {
                    const int i0 = 16 * (tid & 3) + 4 * qd;
                    t4[qd] = *reinterpret_cast<const float4*>(Tf + r * kLd + i0);
                    b4[qd] = *reinterpret_cast<const float4*>(beta_s + i0);
                }
#pragma unroll
                for (int qd = 0; qd < 4; ++qd) {
                    const int i0 = 16 * (tid & 3) + 4 * qd;
                    st_tf32x4(smem, OFF_TP + (i0 >> 5) * KB_TP + sw128_off(r, (i0 & 31) >> 2),
                              (i0 + 0 <= r) ? t4[qd].x * b4[qd].x : 0.f, (i0 + 1 <= r) ? t4[qd].y * b4[qd].y : 0.f,
                              (i0 + 2 <= r) ? t4[qd].z * b4[qd].z : 0.f, (i0 + 3 <= r) ? t4[qd].w * b4[qd].w : 0.f);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ============== delta = T' (V - Y)   (lanes 0-63 of TM_U)
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dtp = tdesc(sb, OFF_TP), dvt = tdesc(sb, OFF_VT);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_tf32_ss(tmem + TM_U, kstep(dtp, KB_TP, s), kstep(dvt, KB_VT, s), ID_N32, s > 0);
            mma_commit(bar_mma);
        }
        mma_pending = true;
        if (!(ok = wait_mma())) break;

        // ============== delta -> delta^T operand (token rows 0-63)
        if (quarter < 2) {   // two warps per lane quarter, 16 value columns each
            float d[16];
            const int c0 = 16 * half;
            tmem_ld16(tm_lane(tmem, quarter, TM_U + c0), d);
            tmem_wait_ld();
            const int r = 32 * quarter + lane;
#pragma unroll
            for (int e = 0; e < 16; ++e) *K_at(smem, OFF_YT, KB_VT, c0 + e, r) = to_tf32(d[e]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ============== O = Z + P delta,  S_next = St + Kb^T delta
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dtp = tdesc(sb, OFF_TP), dkbt = tdesc(sb, OFF_KBT), dyt = tdesc(sb, OFF_YT);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                mma_tf32_ss(tmem + TM_X, kstep(dtp, KB_TP, s), kstep(dyt, KB_VT, s), ID_N32, 1);
                mma_tf32_ss(tmem + TM_S, kstep(dkbt, KB_KBT, s), kstep(dyt, KB_VT, s), ID_N32, 1);
            }
            mma_commit(bar_mma);
        }
        mma_pending = true;

        // ============== while those run: prep of the next chunk (touches neither
        // TP, Kb^T, delta^T nor tensor memory)
        if (has_next) {
            if (!(ok = !__syncthreads_or(!mbar_wait_bounded(bar_load, (c + 1) & 1)))) break;
            load_pending = false;
            lvl_next = prep(Ln);
        }
        if (!(ok = wait_mma())) break;

        // ============== O (token rows in lanes 64-127) -> global
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
    }

    tc_fence_before();
    __syncthreads();
    if (ok && serial) {
        // the recurrence over the whole sequence from the initial state (which this
        // CTA has not written yet), in the now idle shared memory
        if (warp < 4)
            serial_slice(q, k, v, g, beta, bos, eos, H, h, slice, scale, l2norm != 0, scalar_g != 0, s0, sT, state_off,
                         o, nullptr, reinterpret_cast<float*>(smem), tid, 1u);
        __syncthreads();
    } else if (ok) {
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

}  // namespace

namespace {
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
}  // namespace

bool make_token_map(CUtensorMap* map, const void* base, int64_t total_T, int H, bool f32) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t esz = f32 ? 4 : 2;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(total_T)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD) * esz, static_cast<cuuint64_t>(H) * kD * esz};
    cuuint32_t box[3] = {kD, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
               const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_chunk(const PrefillArgs& a, cudaStream_t stream) {
    if (a.N == 0 || a.H == 0) return cudaSuccess;
    if (a.total_T <= 0) return cudaErrorInvalidValue;   // callers route empty batches elsewhere
    static PerDeviceOnce attr_once;
    const cudaError_t attr_err = attr_once.run([] {
        return cudaFuncSetAttribute(kda_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(SMEM_BYTES));
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap mq, mk;
    if (!make_token_map(&mq, a.q, a.total_T, a.H) || !make_token_map(&mk, a.k, a.total_T, a.H))
        return cudaErrorInvalidValue;
    const long long blocks = (long long)a.N * a.H * kSplit;
    return launch_kernel(kda_chunk_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), SMEM_BYTES, stream,
        mq, mk, static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
        static_cast<const __nv_bfloat16*>(a.v), a.g, a.beta, a.cu_seqlens, a.total_T, a.H, a.scale,
        a.l2norm ? 1 : 0, a.scalar_decay ? 1 : 0, a.initial_state, a.final_state, a.o, a.err, a.slots,
        a.num_slots);
}

}  // namespace kda
