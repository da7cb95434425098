// kda_chunk2.cu -- two-pass chunked KDA prefill on Blackwell tensor cores
// (tcgen05 kind::tf32, accumulators in tensor memory, TMA and bulk copies).
//
// The layer's rule (page "GLM-5.3-FLASH", dimsnsums.com, section "How can a
// layer remember without rereading?"):
//     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
//     o_t = scale * S_t^T q_t.
// Evaluated 64 tokens at a time.  For one chunk with entry state S (rows =
// key channels), Gamma_r = g_0 + ... + g_r per channel and Gamma_C its value
// at the chunk's last token, with T' = (I + strict_lower(diag(beta) A))^-1
// diag(beta), A_ri = sum_c k^_rc k^_ic e^(Gamma_rc - Gamma_ic) and P_ri the
// same with scale q^_r (the intra-chunk Gram matrices, taken at the level the
// chunk's decay allows: kda_tile.cuh), the state side has two exact forms:
//   chunk-end form (every channel decays by at most 2^100 over the chunk):
//     Qt = scale q^ e^(Gamma_r - Gamma_C),  Kt = k^ e^(Gamma_r - Gamma_C),
//     Kb = k^ e^(Gamma_C - Gamma_r),  St = Diag(e^Gamma_C) S,
//     W = T' Kt,  U = T' V,  delta = U - W St,
//     O = Qt St + P delta,   S_next = St + Kb^T delta;
//   chunk-start form (any decay; every factor in (0, 1]):
//     Qs = scale q^ e^Gamma_r,  Ks = k^ e^Gamma_r,  same Kb,
//     W = T' Ks,  delta = U - W S,
//     O = Qs S + P delta,   S_next = Diag(e^Gamma_C) S + Kb^T delta.
// Unrolling the per-token rule inside the chunk gives (I + M) delta =
// diag(beta)(V - k^ e^Gamma S) for the rank-one corrections delta_r, from
// which O and S_next follow.  Everything except the last line is independent
// of the state.  Pass 1 (kda_chunk_prep_kernel) therefore runs over all
// (chunk, head) pairs in parallel and writes, per pair, ready-made
// tensor-core operand images of [Q ; W], Kb and P, U, e^Gamma_C and a flag
// naming the form, to scratch.  Pass 2 (kda_chunk_state_kernel) walks the
// chunks of one (sequence, head) in order and only carries the state:
//     (chunk-end form) S^T <- S^T Diag(e^Gamma_C)
//     [Z^T | Y^T] = S^T [Q ; W]^T              (M = 128 value columns, N = 128)
//     (chunk-start form) S^T <- S^T Diag(e^Gamma_C)
//     delta^T = U^T - Y^T,   S_next^T = S^T + delta^T Kb,   O^T = Z^T + delta^T P^T
// The state is kept transposed in tensor memory (lane = value column, column
// = key channel), so it is the A operand of the first products and the
// accumulator of the update, and the readout O^T lands with the value
// column in the lane, which is the contiguous axis of o in global memory.
//
// Operand tiles have 128-byte rows.  K-major tiles (the reduction axis
// contiguous) permute 16-byte chunks by the row index mod 8; MN-major tf32
// tiles (the other axis contiguous), which the tensor core reads with a
// different swizzle, permute 32-byte granules by the row index mod 4.  Pass 1
// writes K (Kt or Ks), Kb and V in the token-row orientation it produces them in and
// lets the products read them MN-major, so no tile is transposed.
//
// Precision: as the fused kernel -- tf32 operands (rounded to nearest),
// fp32 accumulation, fp32 state (decayed on CUDA cores); U is kept in fp32.
#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_tile.cuh"
#include "sm100.cuh"

#include <mutex>

namespace kda {
namespace {

constexpr int kC = 64;
constexpr int kThreads = 256;

// ---- per (chunk, head) operand image in scratch (byte offsets), tiles
// exactly as the state pass holds them in shared memory.
constexpr uint32_t IMG_B1 = 0;        // [Q ; W]: rows 0-63 Q, 64-127 W (token) x 128 channels, K-major,
                                      //   4 K-blocks x 16 KB
constexpr uint32_t IMG_DC = 65536;    // exp(Gamma_C): 128 fp32 (+ 512 B pad)
constexpr uint32_t IMG_KB = 66560;    // Kb: 64 token rows x 128 channels, MN-major, 4 blocks of 32 channels x 8 KB
constexpr uint32_t IMG_P = 99328;     // P: 64 token rows x 64 tokens, K-major, 2 K-blocks x 8 KB
constexpr uint32_t IMG_U = 115712;    // U^T: 128 value rows x 64 tokens fp32, 16-byte chunks permuted as
                                      //   K-major tiles, 2 blocks of 32 tokens x 16 KB
constexpr uint32_t IMG_BYTES = 148480;
constexpr uint32_t KB_B1 = 16384, IMG_BLK = 8192;   // K-block of [Q ; W]; 64 rows x 128 B
constexpr uint32_t IMG_FORM = IMG_DC + 512;   // 16 B: word 0 = 0 for the chunk-end form, 1 for the chunk-start form
constexpr uint32_t B1_COPY = IMG_FORM + 16;   // [Q ; W], exp(Gamma_C) and the form flag in one copy
static_assert(IMG_DC == 4 * 16384 && (B1_COPY - IMG_DC) % 16 == 0, "B1 copy: four 16 KB blocks, then the rest");
constexpr uint32_t B2_COPY = IMG_BYTES - IMG_KB;   // Kb, P and U on one mbarrier phase
static_assert(IMG_KB % 1024 == 0 && IMG_P == IMG_KB + 32768 && IMG_U == IMG_P + 16384 &&
              IMG_BYTES == IMG_U + 32768, "image layout");

__device__ __forceinline__ bool seq_bounds(const int32_t* cu, int n, int64_t total_T, int64_t& bos, int64_t& eos) {
    bos = cu[n];
    eos = cu[n + 1];
    return !(bos < 0 || eos < bos || eos > total_T);
}

// ============================================================ chunk index
// chunk_off[n] = number of 64-token chunks of sequences 0..n-1 (exclusive
// scan), chunk_off[N] = total.  A sequence with inconsistent cu_seqlens gets
// no chunks and sets error bit 1.  Sequences that are each in bounds but
// overlap (cu_seqlens not non-decreasing) can add up to more chunks than the
// scratch holds (max_total): that also sets error bit 1, and both passes
// skip every chunk at or past max_total.  Also clears the ring flags of the
// overlapped mode.  One block.
__global__ void __launch_bounds__(1024) kda_chunk_index_kernel(const int32_t* __restrict__ cu, int N,
                                                               int64_t total_T, int64_t max_total,
                                                               int32_t* __restrict__ chunk_off, uint32_t* err,
                                                               int32_t* __restrict__ zero, int nzero) {
    __shared__ int32_t wsum[32];
    __shared__ int32_t carry_s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < nzero; i += 1024) zero[i] = 0;   // ring flags of the overlapped mode
    if (tid == 0) carry_s = 0;
    __syncthreads();
    for (int base = 0; base < N; base += 1024) {
        const int n = base + tid;
        int32_t cnt = 0;
        if (n < N) {
            int64_t bos, eos;
            if (seq_bounds(cu, n, total_T, bos, eos)) cnt = static_cast<int32_t>((eos - bos + kC - 1) / kC);
            else set_error(err, 1u);
        }
        int32_t x = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int32_t w = wsum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            wsum[lane] = w;
        }
        __syncthreads();
        const int32_t carry = carry_s;
        const int32_t incl = x + (warp > 0 ? wsum[warp - 1] : 0);
        if (n < N) chunk_off[n] = carry + incl - cnt;
        __syncthreads();
        if (tid == 1023) carry_s = carry + incl;
        __syncthreads();
    }
    if (tid == 0) {
        chunk_off[N] = carry_s;
        if (carry_s > max_total) set_error(err, 1u);
    }
}

// ============================================================ pass 1
// Shared memory (byte offsets from a 1024-aligned base).
constexpr uint32_t P_X = 0;          // 64 KB Gram operand: 128 rows (Q-side, K-side) x 128 channels, K-major,
                                     //   4 K-blocks x 16 KB.  After it: [P ; A] staging (levels 1, 2), the
                                     //   triangular-solve scratch (from 0), T' (at P_TP), then P on its way
                                     //   to the image (from 0)
constexpr uint32_t P_TP = 49152;     // 16 KB T': 64 rows (token r) x 64 (token i), K-major, 2 K-blocks x 8 KB
constexpr uint32_t P_KB = 65536;     // 32 KB second Gram operand: 64 rows x 128 channels, K-major, 4 K-blocks
                                     //   x 8 KB; also the TMA destination of the next item's raw q (16 KB)
                                     //   and k (16 KB)
constexpr uint32_t P_KTM = 98304;    // 32 KB Kt or Ks MN-major: 64 token rows x 128 channels, 4 blocks x
                                     //   8 KB (the A operand of W^T)
constexpr uint32_t P_WST = 131072;   // 32 KB W (K-major, 4 K-blocks x 8 KB) on its way to the image; before
                                     //   that the exact Gram's Z table (levels 1, 2)
constexpr uint32_t P_V = 163840;     // 32 KB V MN-major: 64 token rows x 128 values, 4 blocks x 8 KB
                                     //   (V^T for U^T); then U^T on its way out
constexpr uint32_t P_RV = 196608;    // 16 KB raw v (bf16 [64 tokens][128])
constexpr uint32_t P_MISC = 212992;  // beta[64] | xch[8][128] at +1024 | barriers at +5120
constexpr uint32_t P_SMEM = P_MISC + 6144 + 1024;
constexpr uint32_t P_KB_KB = 8192, P_KB_TP = 8192, P_MN_KB = 8192;
// Issues the bulk stores and the ring hand-over.  Its warp (quarter 3) reads
// no P, so the hand-over overlaps the W / U product.  Bulk-store groups per
// item: P (from X), then W and U (from WST and V).
constexpr int kStoreThread = 224;
static_assert(kUtScratchBytes <= P_TP - P_X, "solve scratch");

constexpr uint32_t TP_AP = 0;     // 64 cols: P (lanes 0-63) | A (lanes 64-127)
constexpr uint32_t TP_W = 64;     // 64 cols: W^T (lane = channel, column = token)
constexpr uint32_t TP_U = 128;    // 64 cols: U^T (lane = value column, column = token)
constexpr uint32_t TP_COLS = 256;
constexpr uint32_t ID_N64 = idesc_tf32(128, 64, false, false);
constexpr uint32_t ID_N64_AMN = idesc_tf32(128, 64, true, false);   // A read MN-major

// Overlapped mode (one sequence): the prep role writes each (chunk, head)
// image into a ring of kRing slots per head instead of its own place in the
// scratch, and the two roles hand slots over through flags in global memory:
//   ready(h, s) = c + 1 once chunk c's image sits complete in slot s,
//   done(h)     = number of chunks of head h the state role has read.
// A slot is rewritten only after its previous chunk was read, so the ring
// (kRing x H x IMG_BYTES, 37 MB for 32 heads) stays in L2.
constexpr int kRing = 8;
struct Ring {
    int32_t* ready;
    int32_t* done;
};
// The flags of one head sit in a 128-byte line of their own, so that waiting
// producers and the state CTAs of other heads do not contend for it.
constexpr int kFlagStride = 32;
__device__ __forceinline__ int32_t* ready_flag(const Ring& r, int h, int c) {
    return r.ready + h * kFlagStride + (c & (kRing - 1));
}
__device__ __forceinline__ int32_t* done_flag(const Ring& r, int h) { return r.done + h * kFlagStride; }

// Pass 1 for the work items first, first + stride, ... (item w = chunk w / H
// of head w % H, in the global chunk order of chunk_off).
template <bool RING>
__device__ __forceinline__ void prep_role(const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                          const CUtensorMap* tm_g, const float* __restrict__ g,
                                          const float* __restrict__ beta,
                                          const int32_t* __restrict__ cu, const int32_t* __restrict__ chunk_off,
                                          int N, int H, int64_t max_total, float scale, int l2norm, int scalar_g,
                                          uint8_t* __restrict__ img, uint32_t* err, int64_t first, int64_t stride,
                                          Ring ring) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    float* beta_s = reinterpret_cast<float*>(smem + P_MISC);
    float* xch = reinterpret_cast<float*>(smem + P_MISC + 1024);
    uint64_t* bar_load = reinterpret_cast<uint64_t*>(smem + P_MISC + 5120);
    uint64_t* bar_mma = bar_load + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int64_t total = chunk_off[N];
    const int64_t items = (total < max_total ? total : max_total) * H;
    if (first >= items) return;

    if (warp == 0) {
        tmem_alloc(tmem_slot, TP_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        prefetch_tmap(tm_q);
        prefetch_tmap(tm_k);
        prefetch_tmap(tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // work item w -> chunk gc = w / H of head h = w % H; sequence n = the last
    // one whose first chunk is <= gc (sequences without chunks are skipped).
    // Items are decoded in increasing order, stride apart: (gc, h) advances by
    // (stride / H, stride % H) with a carry, and the sequence search goes on
    // from the previous item's sequence.
    struct Item {
        int64_t t0, gc;
        int L, h, c;   // c: chunk index inside its sequence
    };
    const int64_t step_gc = stride / H;
    const int step_h = static_cast<int>(stride - step_gc * H);
    int seq = 0;
    auto advance = [&](Item p) {
        p.gc += step_gc;
        p.h += step_h;
        if (p.h >= H) {
            p.h -= H;
            ++p.gc;
        }
        return p;
    };
    auto decode = [&](Item it) {
        while (seq + 1 < N && chunk_off[seq + 1] <= it.gc) ++seq;
        const int lo = seq;
        it.c = static_cast<int>(it.gc - chunk_off[lo]);
        it.t0 = cu[lo] + static_cast<int64_t>(it.c) * kC;
        const int64_t rem = cu[lo + 1] - it.t0;
        it.L = static_cast<int>(rem < kC ? rem : (int64_t)kC);
        return it;
    };
    // the item's image: its own place in the scratch, or its head's ring slot
    auto image_of = [&](const Item& it) {
        const size_t slot = RING ? static_cast<size_t>(it.h) * kRing + (it.gc & (kRing - 1))
                                 : static_cast<size_t>(it.gc) * H + it.h;
        return img + slot * IMG_BYTES;
    };
    // ring mode: the image of an item (Q, Kb, exp(Gamma_C) and the form written with
    // plain stores before the item's block barriers, the rest by bulk stores)
    // is announced by the store thread once those bulk stores have completed:
    // a proxy fence, then a gpu-scope release, which also covers the plain
    // stores of the other threads (ordered before it by the barriers).  That
    // happens when the next item's rows reach their decay sums, or before the
    // store thread blocks on a slot.
    int32_t* pub_flag = nullptr;
    int32_t pub_val = 0;
    auto publish = [&]() {
        bulk_wait_all();
        if (RING && pub_flag) {
            fence_proxy_async_global();
            st_release_gpu(pub_flag, pub_val);
            pub_flag = nullptr;
        }
    };
    // store thread: done[] of the item's head, read one item ahead
    int32_t done_seen = 0;
    // q, k, v and g are read once: evict them first, ahead of the ring's images
    const uint64_t stream_policy = l2_evict_first();
    float greg[8][4];
    float breg;
    auto prefetch = [&](const Item& it) {
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int r = 8 * warp + m;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < it.L) {
                if (scalar_g) {
                    const float gs = __ldg(g + (size_t)(it.t0 + r) * H + it.h);
                    x = make_float4(gs, gs, gs, gs);
                } else {
                    x = ldg_hint(reinterpret_cast<const float4*>(g + ((size_t)(it.t0 + r) * H + it.h) * kD + 4 * lane),
                                 stream_policy);
                }
            }
            greg[m][0] = x.x; greg[m][1] = x.y; greg[m][2] = x.z; greg[m][3] = x.w;
        }
        breg = 0.f;
        if (tid < it.L) breg = __ldg(beta + (size_t)(it.t0 + tid) * H + it.h);
    };
    auto issue_load = [&](const Item& it) {
        mbar_arrive_expect_tx(bar_load, 3u * kC * kD * 2u);
        const int32_t t0 = static_cast<int32_t>(it.t0);
        tma_load_3d_hint(smem + P_KB, tm_q, bar_load, 0, it.h, t0, stream_policy);
        tma_load_3d_hint(smem + P_KB + kC * kD * 2, tm_k, bar_load, 0, it.h, t0, stream_policy);
        tma_load_3d_hint(smem + P_RV, tm_v, bar_load, 0, it.h, t0, stream_policy);
    };

    bool ok = true;
    uint32_t load_parity = 0, mma_phase = 0;
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

    int64_t w = first;
    Item pos2;   // position (gc, h) of the item two ahead
    pos2.gc = first / H;
    pos2.h = static_cast<int>(first - pos2.gc * H);
    Item cur = decode(pos2);
    pos2 = advance(pos2);
    Item nxt = w + stride < items ? decode(pos2) : cur;
    pos2 = advance(pos2);
    Item nxt2 = w + 2 * stride < items ? decode(pos2) : cur;   // only for an L2 prefetch
    if (tid == 0) issue_load(cur);
    load_pending = true;
    prefetch(cur);

    for (; ok && w < items; w += stride) {
        const int64_t wn = w + stride, w2 = wn + stride;
        const bool has_next = wn < items, has_next2 = w2 < items;
        uint8_t* im = image_of(cur);
        const int L = cur.L;

        // ring mode: the slot must have been read by the state role first.  A
        // producer never blocks on it while holding an unannounced image (the
        // state role that it waits for may need exactly that image).
        bool slot_free = true;
        const int32_t gcur = static_cast<int32_t>(cur.gc);   // the head's ring counts global chunks
        if (RING && tid == kStoreThread && gcur >= kRing && done_seen < gcur - kRing + 1 &&
            ld_acquire_gpu(done_flag(ring, cur.h)) < gcur - kRing + 1) {
            publish();
            slot_free = wait_flag_ge(done_flag(ring, cur.h), gcur - kRing + 1, 1u << 20, 256);
        }
        // the previous item's P has left X, which is rewritten below
        if (tid == kStoreThread) bulk_wait_read_but<1>();
        if (!(ok = !__syncthreads_or(!mbar_wait_bounded(bar_load, load_parity) || !slot_free))) break;
        load_pending = false;
        load_parity ^= 1;

        // ============== prep.  Two forms of the state-side operands, chosen by the chunk's
        // Gram level (kda_tile.cuh), which the image records for the state role:
        //   chunk-end form (level 0, every channel decays by at most 2^kSafeLog2 over the
        //   chunk): Qt = q^ 2^(Gamma_r - Gamma_C), Kt = k^ 2^(Gamma_r - Gamma_C) (<= 2^100),
        //   Kb = k^ 2^(Gamma_C - Gamma_r); the state role decays the state to the chunk end
        //   first and MMA1 reads the decayed state;
        //   chunk-start form (levels 1, 2, any decay): Qs = q^ 2^Gamma_r, Ks = k^ 2^Gamma_r,
        //   same Kb (every factor <= 1); MMA1 reads the state at the chunk start and the
        //   state role decays it afterwards.
        // Either way: Q -> image rows 0-63 of [Q ; W] (K-major), K -> KTM (MN-major, for W),
        // Kb -> image (MN-major), 2^Gamma_C and the form flag -> image.  The Gram operands in
        // X (128 rows, Q-side then K-side) and KB (64 rows), both K-major:
        //   level 0: [Qt ; Kt] and Kb, tf32 (one tensor-core product through the chunk end);
        //   level 1: [q^ X ; k^ X] (fp32) and k^ Y (tf32) (block references);
        //   level 2: [q^ ; k^] and Gamma, fp32.
        // A warp stores four whole 128-byte rows of the image at a time.
        int level = 0;
        {
            // Gamma_C, and the block ends rho_{a-1}, rho_a of the thread's block a = warp / 2
            // (level 1); the full block-end table is rebuilt from xch after the rows
            float4 gc, bprev, bcur;
            auto setup = [&](const ChunkChannels& cc, int lvl) {
                // the previous item's W and U bulk stores have had the row
                // normalisation and the decay sums to complete: announce its image
                if (tid == kStoreThread) publish();
                level = lvl;
                gc = cc.rho[3];
                bprev = cc.bstart;
                bcur = cc.bend;
            };
            // the six stores of one row and 4 channels
            auto put = [&](int r, int kbi, int ch, float4 xq, float4 xk, float4 y, float4 k4, float4 q4, float4 b4) {
                *reinterpret_cast<float4*>(smem + P_X + kbi * KB_B1 + sw128_off(r, ch)) = xq;
                *reinterpret_cast<float4*>(smem + P_X + kbi * KB_B1 + sw128_off(64 + r, ch)) = xk;
                *reinterpret_cast<float4*>(smem + P_KB + kbi * P_KB_KB + sw128_off(r, ch)) = y;
                *reinterpret_cast<float4*>(smem + P_KTM + kbi * P_MN_KB + sw32g_off(r, ch)) = k4;
                *reinterpret_cast<float4*>(im + IMG_B1 + kbi * KB_B1 + sw128_off(r, ch)) = q4;
                *reinterpret_cast<float4*>(im + IMG_KB + kbi * IMG_BLK + sw32g_off(r, ch)) = b4;
            };
            // level 0 (the common case) in a pass of its own, without the other levels'
            // branches; a chunk of level 1 or 2 runs the rows again with the general emit
            prep_chunk_rows<0>(smem + P_KB, smem + P_KB + kC * kD * 2, greg, xch, L, scale, l2norm != 0, setup,
                               [&](int r, int kbi, int ch, float4 qn, float4 kn, float4 gr) {
                const float4 a = sub4(gr, gc);   // >= 0, at most kSafeLog2 at this level
                const float4 E = ex2x4(a), F = ex2x4(make_float4(-a.x, -a.y, -a.z, -a.w));
                const float4 qt = mul4(qn, E), kt = mul4(kn, E), kb = mul4(kn, F);
                const float4 q4 = tf32x4(qt.x, qt.y, qt.z, qt.w), k4 = tf32x4(kt.x, kt.y, kt.z, kt.w),
                             b4 = tf32x4(kb.x, kb.y, kb.z, kb.w);
                put(r, kbi, ch, q4, k4, b4, k4, q4, b4);
            });
            if (level != 0) {
                __syncthreads();   // every warp is past the first pass's reads of xch
                prep_chunk_rows(smem + P_KB, smem + P_KB + kC * kD * 2, greg, xch, L, scale, l2norm != 0, setup,
                                [&](int r, int kbi, int ch, float4 qn, float4 kn, float4 gr) {
                    // chunk-start form (every factor <= 1)
                    const float4 e0 = ex2x4(gr), f = ex2x4(sub4(gc, gr));
                    const float4 qs = mul4(qn, e0), ks = mul4(kn, e0), kb = mul4(kn, f);
                    const float4 q4 = tf32x4(qs.x, qs.y, qs.z, qs.w), k4 = tf32x4(ks.x, ks.y, ks.z, ks.w),
                                 b4 = tf32x4(kb.x, kb.y, kb.z, kb.w);
                    if (level == 1) {   // block references: X = 2^(Gamma_r - rho_{a-1}), Y = 2^(rho_a - Gamma_r)
                        const float4 X = ex2x4(sub4(gr, bprev)), Y = ex2x4(sub4(bcur, gr));
                        const float4 ky = mul4(kn, Y);
                        put(r, kbi, ch, mul4(qn, X), mul4(kn, X), tf32x4(ky.x, ky.y, ky.z, ky.w), k4, q4, b4);
                    } else {
                        put(r, kbi, ch, qn, kn, gr, k4, q4, b4);
                    }
                });
            }
            if (warp == 0) *reinterpret_cast<float4*>(im + IMG_DC + 16 * lane) = ex2x4(gc);
            if (tid == 64)
                *reinterpret_cast<float4*>(im + IMG_FORM) = make_float4(level != 0 ? 1.f : 0.f, 0.f, 0.f, 0.f);
            if (tid < kC) beta_s[tid] = breg;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ============== [P ; A]: level 0 by one tensor-core product [Qt ; Kt] x Kb^T
        // (P in lanes 0-63, A in lanes 64-127 of TP_AP), levels 1 and 2 on CUDA cores and
        // mma.sync (gram_exact), staged into the same tensor-memory columns
        if (level == 0 && tid == 0) {
            tc_fence_after();
            const uint64_t dx = tdesc(sb, P_X), dkb = tdesc(sb, P_KB);
#pragma unroll
            for (int s = 0; s < 16; ++s)
                mma_tf32_ss(tmem + TP_AP, kstep(dx, KB_B1, s), kstep(dkb, P_KB_KB, s), ID_N64, s > 0);
            mma_commit(bar_mma);
        }
        if (level == 0) mma_pending = true;
        if (level != 0 && warp == 0) {
            // block ends -> [4][128] table in xch, in place: xch row w holds the Gamma sum of
            // warp w's 8 rows, and rho_a = the sum over warps 0 .. 2a + 1, added in the order
            // (and so to the same floats) as in the rows' prefix
            float4 t[8];
#pragma unroll
            for (int v = 0; v < 8; ++v) t[v] = *reinterpret_cast<const float4*>(xch + v * kD + 4 * lane);
            float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                run = make_float4(run.x + t[v].x, run.y + t[v].y, run.z + t[v].z, run.w + t[v].w);
                if (v & 1) *reinterpret_cast<float4*>(xch + (v >> 1) * kD + 4 * lane) = run;
            }
        }
        // ============== meanwhile: V (MN-major; bf16 is exact in tf32) from the raw
        // tile, rows past L zero; a 32-byte granule holds the 8 values of a raw chunk
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
            const int id = qd * kThreads + tid, r = id >> 4, j = id & 15;   // row r, values 8 j .. 8 j + 7
            uint4 u = make_uint4(0u, 0u, 0u, 0u);
            if (r < L) u = *reinterpret_cast<const uint4*>(smem + P_RV + r * (kD * 2) + 16 * j);
            uint8_t* dst = smem + P_V + (j >> 2) * P_MN_KB;
            *reinterpret_cast<float4*>(dst + sw32g_off(r, 2 * (j & 3))) =
                make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                            __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
            *reinterpret_cast<float4*>(dst + sw32g_off(r, 2 * (j & 3) + 1)) =
                make_float4(__uint_as_float(u.z << 16), __uint_as_float(u.z & 0xFFFF0000u),
                            __uint_as_float(u.w << 16), __uint_as_float(u.w & 0xFFFF0000u));
        }
        fence_proxy_async_smem();
        // KB and RV are free once the Gram inputs are read: stage the next item's raw
        // q, k, v, and bring the item after it (its q, k, v and g) into L2 so that its
        // loads find it there
        auto next_loads = [&]() {
            if (tid == 0 && has_next) {
                issue_load(nxt);
                if (has_next2) {
                    const int32_t t2 = static_cast<int32_t>(nxt2.t0);
                    tma_prefetch_3d(tm_q, 0, nxt2.h, t2);
                    tma_prefetch_3d(tm_k, 0, nxt2.h, t2);
                    tma_prefetch_3d(tm_v, 0, nxt2.h, t2);
                    if (!scalar_g) tma_prefetch_3d(tm_g, 0, nxt2.h, t2);
                }
            }
        };
        if (level == 0) {
            if (!(ok = wait_mma())) break;
            next_loads();
        } else {
            __syncthreads();   // the block-end table is written
            float* st = reinterpret_cast<float*>(smem + P_X);
            gram_exact(smem + P_X, KB_B1, smem + P_KB, P_KB_KB, xch, reinterpret_cast<float*>(smem + P_WST), st,
                       level, tid, next_loads);
            // [P ; A] -> tensor memory: lane quarter q, value columns 32 * half ..
            {
                float acc[32];
                const float* row = st + (32 * quarter + lane) * kStLd + 32 * half;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 x = *reinterpret_cast<const float4*>(row + 4 * j);
                    acc[4 * j] = x.x; acc[4 * j + 1] = x.y; acc[4 * j + 2] = x.z; acc[4 * j + 3] = x.w;
                }
                tmem_st32(tm_lane(tmem, quarter, TP_AP + 32 * half), acc);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
        }
        load_pending = has_next;

        // ============== A -> M = strict_lower(beta A) (fp32, in X); P stays in TMEM
        float* Mf = reinterpret_cast<float*>(smem + P_X);
        float* Tf = Mf + 64 * kLd;
        float* Y1 = Tf + 64 * kLd;
        float* Y2 = Y1 + 2 * 16 * kLd1;
        if (quarter >= 2) {
            float acc[32];
            tmem_ld32(tm_lane(tmem, quarter, TP_AP + 32 * half), acc);
            tmem_wait_ld();
            const int r = 32 * quarter + lane - 64;
            const float br = beta_s[r];
            float* mrow = Mf + r * kLd + 32 * half;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i0 = 32 * half + 4 * j;
                *reinterpret_cast<float4*>(mrow + 4 * j) =
                    make_float4((i0 + 0 < r) ? br * acc[4 * j + 0] : 0.f, (i0 + 1 < r) ? br * acc[4 * j + 1] : 0.f,
                                (i0 + 2 < r) ? br * acc[4 * j + 2] : 0.f, (i0 + 3 < r) ? br * acc[4 * j + 3] : 0.f);
            }
        }
        tc_fence_before();
        __syncthreads();

        // ============== T = (I + M)^-1, T' = T diag(beta) -> TP (tf32 operand, rows r, K = i)
        ut_inverse64(Mf, Tf, Y1, Y2, tid, [] {});
        {
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
                st_tf32x4(smem, P_TP + (i0 >> 5) * P_KB_TP + sw128_off(r, (i0 & 31) >> 2),
                          (i0 + 0 <= r) ? t4[qd].x * b4[qd].x : 0.f, (i0 + 1 <= r) ? t4[qd].y * b4[qd].y : 0.f,
                          (i0 + 2 <= r) ? t4[qd].z * b4[qd].z : 0.f, (i0 + 3 <= r) ? t4[qd].w * b4[qd].w : 0.f);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ============== W^T = K^T T'^T,  U^T = V^T T'^T  (K and V read MN-major)
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dkt = sdesc_mn32(sb + P_KTM, P_MN_KB), dv = sdesc_mn32(sb + P_V, P_MN_KB);
            const uint64_t dtp = tdesc(sb, P_TP);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                mma_tf32_ss(tmem + TP_W, mn_kstep(dkt, s), kstep(dtp, P_KB_TP, s), ID_N64_AMN, s > 0);
                mma_tf32_ss(tmem + TP_U, mn_kstep(dv, s), kstep(dtp, P_KB_TP, s), ID_N64_AMN, s > 0);
            }
            mma_commit(bar_mma);
        }
        mma_pending = true;
        if (has_next) prefetch(nxt);
        if (tid == kStoreThread) {
            publish();   // (announced already; the call only covers the last item of a loop exit)
            if (RING && has_next) done_seen = ld_relaxed_gpu(done_flag(ring, nxt.h));
        }
        // ============== meanwhile P (lower incl., tf32, K-major) from TMEM -> X (free
        // since T' was built): lanes 0-31 by warp 4, lanes 32-63 by warps 1 and 5
        if (warp == 1 || warp == 4 || warp == 5) {
            const int r = 32 * quarter + lane;
            const int hb = warp == 5 ? 1 : 0, he = warp == 1 ? 1 : 2;
            for (int hh = hb; hh < he; ++hh) {
                float acc[32];
                tmem_ld32(tm_lane(tmem, quarter, TP_AP + 32 * hh), acc);
                tmem_wait_ld();
                uint8_t* dst = smem + P_X + hh * IMG_BLK;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int i0 = 32 * hh + 4 * j;
                    *reinterpret_cast<float4*>(dst + sw128_off(r, j)) =
                        tf32x4((i0 + 0 <= r) ? acc[4 * j + 0] : 0.f, (i0 + 1 <= r) ? acc[4 * j + 1] : 0.f,
                               (i0 + 2 <= r) ? acc[4 * j + 2] : 0.f, (i0 + 3 <= r) ? acc[4 * j + 3] : 0.f);
                }
            }
        }
        fence_proxy_async_smem();
        if (!(ok = wait_mma())) break;
        if (tid == kStoreThread) {
            bulk_store(im + IMG_P, smem + P_X, 2 * IMG_BLK);
            bulk_commit();
        }

        // ============== W (tf32, K-major [token][channel]) -> WST and U^T (fp32,
        // row = value column) -> V (its product is done); then both to the image
        {
            float acc[32];
            const int c = 32 * quarter + lane;   // channel (W) or value column (U)
            tmem_ld32(tm_lane(tmem, quarter, TP_W + 32 * half), acc);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) *K_at(smem, P_WST, IMG_BLK, 32 * half + j, c) = to_tf32(acc[j]);
            tmem_ld32(tm_lane(tmem, quarter, TP_U + 32 * half), acc);
            tmem_wait_ld();
            uint8_t* ut = smem + P_V + half * (2 * IMG_BLK);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<float4*>(ut + sw128_off(c, j)) =
                    make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == kStoreThread) {
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
                bulk_store(im + IMG_B1 + kb * KB_B1 + IMG_BLK, smem + P_WST + kb * IMG_BLK, IMG_BLK);
            bulk_store(im + IMG_U, smem + P_V, 4 * IMG_BLK);
            bulk_commit();
            if (RING) {
                pub_flag = ready_flag(ring, cur.h, static_cast<int>(cur.gc));
                pub_val = static_cast<int32_t>(cur.gc) + 1;
            }
        }
        cur = nxt;
        nxt = nxt2;
        pos2 = advance(pos2);
        if (w2 + stride < items) nxt2 = decode(pos2);
    }

    if (tid == kStoreThread) {
        bulk_wait_all();
        if (ok) publish();
    }
    tc_fence_before();
    __syncthreads();
    if (!ok && tid == 0) {
        set_error(err, 2u);
        if (load_pending) mbar_wait_bounded(bar_load, load_parity, 1u << 16);
        if (mma_pending) mbar_wait_bounded(bar_mma, mma_phase, 1u << 16);
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TP_COLS);
    }
}

// ============================================================ pass 2
// The state pass keeps the image layout: shared-memory offsets equal image offsets.
constexpr uint32_t S_B1 = 0;          // 64 KB [Q ; W] of the current chunk
constexpr uint32_t S_DC = 65536;      // exp(Gamma_C) and the form flag, copied with [Q ; W]
constexpr uint32_t S_KB = 66560;      // 32 KB Kb (MN-major), copied with U, then
constexpr uint32_t S_P = 99328;       //   16 KB P (K-major)
constexpr uint32_t S_U = 115712;      // 32 KB U^T
constexpr uint32_t S_DT = 148480;     // 32 KB delta^T: 128 value rows x 64 tokens, 2 K-blocks x 16 KB
constexpr uint32_t S_OS = 181248;     // 32 KB O of the previous chunk ([token][value] fp32), TMA store source
constexpr uint32_t S_MISC = 214016;   // barriers, TMEM slot
constexpr uint32_t S_SMEM = S_MISC + 1024 + 1024;
static_assert(S_B1 == IMG_B1 && S_DC == IMG_DC && S_KB == IMG_KB && S_P == IMG_P && S_U == IMG_U &&
              S_DT == IMG_BYTES && S_DT % 1024 == 0, "layout");

constexpr uint32_t TS_S = 0;      // 128 cols: S^T fp32 (lane = value column, column = key channel)
constexpr uint32_t TS_Z = 128;    // 64 cols: Z^T, then O^T (column = token) of even chunks; Y^T follows;
                                  //   odd chunks use the set 256 columns on (384 - 511)
constexpr uint32_t TS_COLS = 512;
constexpr uint32_t ID_N128 = idesc_tf32(128, 128, false, false);
constexpr uint32_t ID_N128_BMN = idesc_tf32(128, 128, false, true);   // B read MN-major
constexpr int kImgThread = 32;    // waits for the next chunk's image during MMA1 and copies it in
constexpr int kOutThread = 128;   // issues the O stores, the L2 prefetches and the ring hand-back
                                  // (first thread of the O warps; not the MMA thread)

// Pass 2 for head h over the sequences n_begin .. n_end - 1.  Per chunk c
// (k = c % 2 selects one of two Z/Y column sets in TMEM):
//   decay:  S = Diag(e^Gamma_C) S in place in TMEM (fp32, all warps): here for the
//           chunk-end form, after MMA1 for the chunk-start form
//   MMA1:   [Z_k | Y_k] = S^T [Q ; W]^T          (A = the state in TMEM, read as
//           tf32; B = [Q ; W])
//           meanwhile O of chunk c-1 (set k^1) is read out and staged
//   delta:  delta^T = U^T - Y_k^T                                  (all warps)
//   MMA2a:  S^T += delta^T Kb   (Kb read MN-major; the only product the next chunk waits for)
//   MMA2b:  Z_k^T += delta^T P^T  = O^T of chunk c, read out during chunk c+1
template <bool RING>
__device__ __forceinline__ void state_role(const CUtensorMap* tm_o, const uint8_t* __restrict__ img,
                                           const int32_t* __restrict__ chunk_off, const int32_t* __restrict__ cu,
                                           int64_t total_T, int H, int64_t max_total, const float* s0, float* sT,
                                           float* __restrict__ o, uint32_t* err, const int32_t* __restrict__ slots,
                                           int num_slots, int n_begin, int n_end, int h, Ring ring) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    uint64_t* bar_b1 = reinterpret_cast<uint64_t*>(smem + S_MISC);
    uint64_t* bar_b2 = bar_b1 + 1;
    uint64_t* bar_mma = bar_b1 + 2;   // MMA1 and MMA2a of every chunk
    uint64_t* bar_o = bar_b1 + 3;     // MMA2b of every chunk
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_b1 + 4);
    const float* dc_s = reinterpret_cast<const float*>(smem + S_DC);
    float* dc_keep = reinterpret_cast<float*>(smem + S_MISC + 512);   // 2^Gamma_C of the current chunk

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int e = 32 * quarter + lane;   // value column of this thread's TMEM lane

    if (warp == 0) {
        tmem_alloc(tmem_slot, TS_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_b1, 1);
        mbar_init(bar_b2, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_o, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // state carried across the sequences of this CTA: mbarrier phases follow the
    // running chunk count `base` (one B1, one B2 and one MMA2b phase per chunk,
    // two phases of bar_mma), and the in-flight copies and products with the
    // running chunk index they belong to
    uint32_t base = 0, mma_phase = 0;
    bool ok = true, img_ok = true;   // img_ok: thread 0's image waits did not give up
    bool b1_pending = false, b2_pending = false, mma_pending = false, o_pending = false;
    int b1_chunk = 0, b2_chunk = 0;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
        return !__syncthreads_or(!mbar_wait_bounded(bar, parity));
    };
    auto zcol = [](int c) { return TS_Z + 256u * static_cast<uint32_t>(c & 1); };   // Z of chunk c; Y follows
    // S <- Diag(d) S in place in TMEM (fp32): key channels 64 * half .. of value column e;
    // the caller waits for the stores (tmem_wait_st) before the next product reads S
    auto decay_state = [&](const float* d) {
        float st[2][32];
#pragma unroll
        for (int part = 0; part < 2; ++part) tmem_ld32(tm_lane(tmem, quarter, TS_S + 64 * half + 32 * part), st[part]);
        tmem_wait_ld();
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            const int c0 = 64 * half + 32 * part;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 d4 = *reinterpret_cast<const float4*>(d + c0 + 4 * j);
                st[part][4 * j] *= d4.x; st[part][4 * j + 1] *= d4.y;
                st[part][4 * j + 2] *= d4.z; st[part][4 * j + 3] *= d4.w;
            }
            tmem_st32(tm_lane(tmem, quarter, TS_S + c0), st[part]);
        }
    };

    for (int n = n_begin; ok && n < n_end; ++n) {
    __syncthreads();   // the previous sequence's final state has left tensor memory
    int64_t bos, eos;
    if (!seq_bounds(cu, n, total_T, bos, eos)) continue;   // flagged by the index kernel
    const int64_t sidx = slots ? static_cast<int64_t>(slots[n]) : static_cast<int64_t>(n);
    const int nch = static_cast<int>((eos - bos + kC - 1) / kC);
    const int64_t gc0 = chunk_off[n];
    // a sequence skipped below still has its chunks' images made by the prep role (as far
    // as the scratch reaches); in ring mode they are handed back unread, so that the
    // producers waiting for those slots go on
    auto drain = [&]() -> bool {
        bool good = true;
        if (RING && tid == kOutThread) {
            const int64_t last = gc0 + nch < max_total ? gc0 + nch : max_total;
            for (int64_t gcx = gc0; good && gcx < last; ++gcx) {
                good = wait_flag_ge(ready_flag(ring, h, static_cast<int>(gcx)), static_cast<int>(gcx + 1));
                if (good) st_relaxed_gpu(done_flag(ring, h), static_cast<int>(gcx + 1));
            }
        }
        return !__syncthreads_or(!good);
    };
    if (slots && (sidx < 0 || sidx >= num_slots)) {
        if (tid == 0 && h == 0) set_error(err, 4u);
        if (!(ok = drain())) break;
        continue;
    }
    if (gc0 + nch > max_total) {   // overlapping sequences overflowed the scratch: flagged above
        if (!(ok = drain())) break;
        continue;
    }
    auto image = [&](int c) {
        const size_t slot = RING ? static_cast<size_t>(h) * kRing + ((gc0 + c) & (kRing - 1))
                                 : static_cast<size_t>(gc0 + c) * H + h;
        return img + slot * IMG_BYTES;
    };
    // ring mode: chunk c's image must be complete before its first copy is issued
    auto await_image = [&](int c) -> bool {
        if (!RING) return true;
        const bool good = wait_flag_ge(ready_flag(ring, h, static_cast<int>(gc0 + c)), static_cast<int>(gc0 + c + 1));
        fence_proxy_async_global();
        return good;
    };
    img_ok = true;


    const size_t state_off = ((size_t)sidx * H + h) * kD * kD;

    // initial state, transposed: lane e = value column, columns = key rows 64*half ..
    {
        float r[32];
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            const int c0 = 64 * half + 32 * part;
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = s0 ? s0[state_off + (size_t)(c0 + j) * kD + e] : 0.f;
            tmem_st32(tm_lane(tmem, quarter, TS_S + c0), r);
        }
        tmem_wait_st();
    }
    auto load_b1 = [&](int c) {
        mbar_arrive_expect_tx(bar_b1, B1_COPY);
        const uint8_t* src = image(c);
#pragma unroll
        for (int p = 0; p < 4; ++p) bulk_load(smem + S_B1 + p * 16384, src + p * 16384, 16384, bar_b1);
        bulk_load(smem + S_DC, src + IMG_DC, B1_COPY - IMG_DC, bar_b1);
    };
    // Kb, P and U in two steps on one mbarrier phase (the first step
    // registers all the bytes): Kb and U as soon as MMA2a of the previous
    // chunk is done, P once MMA2b (which reads P) is done
    auto load_b2_kb_u = [&](int c) {
        mbar_arrive_expect_tx(bar_b2, B2_COPY);
        const uint8_t* src = image(c);
        bulk_load(smem + S_KB, src + IMG_KB, 4 * IMG_BLK, bar_b2);
        bulk_load(smem + S_U, src + IMG_U, 4 * IMG_BLK, bar_b2);
    };
    auto load_b2_p = [&](int c) { bulk_load(smem + S_P, image(c) + IMG_P, 2 * IMG_BLK, bar_b2); };
    auto load_b2 = [&](int c) {
        load_b2_kb_u(c);
        load_b2_p(c);
    };
    if (tid == 0 && nch > 0) {
        img_ok = await_image(0);
        if (img_ok) {
            load_b1(0);
            load_b2(0);
        }
    }
    ok = !__syncthreads_or(!img_ok);
    if (!ok) break;
    b1_pending = b2_pending = nch > 0;
    b1_chunk = b2_chunk = static_cast<int>(base);
    if (!RING && tid == kOutThread && nch > 1) prefetch_l2(image(1), IMG_BYTES);

    int64_t t_prev = bos;
    for (int c = 0; c < nch; ++c) {
        const int64_t t0 = bos + (int64_t)c * kC;
        const int L = static_cast<int>(eos - t0 < kC ? eos - t0 : (int64_t)kC);

        // ---- the state at the chunk start is in TMEM once MMA2a of chunk c-1 is done
        if (c > 0) {
            if (!(ok = wait_all(bar_mma, mma_phase))) break;
            mma_phase ^= 1;
            mma_pending = false;
            tc_fence_after();
            if (tid == 0) load_b2_kb_u(c);
            b2_pending = true;
            b2_chunk = static_cast<int>(base) + c;
        }
        if (!RING && tid == kOutThread && c + 2 < nch) prefetch_l2(image(c + 2), IMG_BYTES);
        if (tid == kOutThread) bulk_wait_read();   // the O staging tile is rewritten below
        // [Q ; W], 2^Gamma_C and the form flag of chunk c have landed.  Chunk-end form:
        // the state is decayed to the chunk end now and MMA1 reads it decayed.  Chunk-start
        // form: MMA1 reads the state as it is and the decay follows MMA1, so 2^Gamma_C is
        // kept aside (the next chunk's copy lands on top of it before then).
        const bool b1_ok = mbar_wait_bounded(bar_b1, (base + c) & 1);
        const bool start_form = b1_ok && dc_s[kD] != 0.f;   // the same word for every thread
        if (b1_ok && !start_form) decay_state(dc_s);
        if (b1_ok && start_form && tid < kD / 4)
            reinterpret_cast<float4*>(dc_keep)[tid] = reinterpret_cast<const float4*>(dc_s)[tid];
        tmem_wait_st();
        tc_fence_before();
        if (!(ok = !__syncthreads_or(!b1_ok))) break;
        b1_pending = false;

        // ---- MMA1: [Z_k^T | Y_k^T] = S^T [Q ; W]^T (the state, decayed or not by the
        // form, read by the tensor core as tf32: the low mantissa bits are dropped;
        // measured on the CPU against the fp64 oracle: no change in the error of o or S)
        if (tid == 0) {
            tc_fence_after();
            const uint64_t db = tdesc(sb, S_B1);
#pragma unroll
            for (int s = 0; s < 16; ++s)
                mma_tf32_ts(tmem + zcol(c), tmem + TS_S + 8 * s, kstep(db, KB_B1, s), ID_N128, s > 0);
            mma_commit(bar_mma);
        }
        mma_pending = true;
        // meanwhile: the next chunk's image is awaited (its copy waits for MMA1,
        // which reads the tile it lands in), off the issuing thread
        if (tid == kImgThread && c + 1 < nch) img_ok = await_image(c + 1);
        // and (warps 4-7) O of chunk c-1 (a full chunk) goes into the staging
        // tile; its product MMA2b also read P, so chunk c's copy of P waits for it
        bool o_ok = true;
        if (c > 0 && half == 1) {
            o_ok = mbar_wait_bounded(bar_o, (base + c - 1) & 1);
            if (o_ok) {
                tc_fence_after();
                if (tid == kOutThread) load_b2_p(c);
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    float acc[32];
                    tmem_ld32(tm_lane(tmem, quarter, zcol(c - 1) + 32 * part), acc);
                    tmem_wait_ld();
                    float* dst = reinterpret_cast<float*>(smem + S_OS) + (32 * part) * kD + e;
#pragma unroll
                    for (int j = 0; j < 32; ++j) dst[j * kD] = acc[j];
                }
            }
            fence_proxy_async_smem();
        }
        tc_fence_before();
        if (!(ok = !__syncthreads_or(!mbar_wait_bounded(bar_mma, mma_phase) || !o_ok))) break;
        mma_phase ^= 1;
        mma_pending = false;
        if (c > 0) o_pending = false;
        tc_fence_after();
        if (c > 0 && tid == kOutThread) {   // O of chunk c-1 leaves by one TMA store
            tma_store_3d_hint(tm_o, smem + S_OS, 0, h, static_cast<int32_t>(t_prev), l2_evict_first());
            bulk_commit();
        }
        if (tid == kImgThread && c + 1 < nch && img_ok) load_b1(c + 1);
        b1_pending = c + 1 < nch;
        b1_chunk = static_cast<int>(base) + c + 1;

        // ---- chunk-start form: the decay, now that MMA1 (its last reader) is done;
        // delta^T = U^T - Y_k^T (tf32 operand, row = value column, K = token);
        // U^T came with Kb
        if (start_form) decay_state(dc_keep);
        const bool b2_ok = mbar_wait_bounded(bar_b2, (base + c) & 1);
        if (b2_ok) {
            float y[32];
            tmem_ld32(tm_lane(tmem, quarter, zcol(c) + 64 + 32 * half), y);
            const uint8_t* us = smem + S_U + half * (2 * IMG_BLK);
            float u[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 x = *reinterpret_cast<const float4*>(us + sw128_off(e, j));
                u[4 * j] = x.x; u[4 * j + 1] = x.y; u[4 * j + 2] = x.z; u[4 * j + 3] = x.w;
            }
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<float4*>(K_at(smem, S_DT, 16384, e, 32 * half + 4 * j)) =
                    tf32x4(u[4 * j] - y[4 * j], u[4 * j + 1] - y[4 * j + 1], u[4 * j + 2] - y[4 * j + 2],
                           u[4 * j + 3] - y[4 * j + 3]);
        }
        tmem_wait_st();   // (chunk-start form) the decayed state is in place before MMA2a accumulates onto it
        fence_proxy_async_smem();
        tc_fence_before();
        if (!(ok = !__syncthreads_or(!b2_ok || !img_ok))) {
            b1_pending = b1_pending && img_ok;
            break;
        }
        b2_pending = false;
        // chunk c's slot is read: both copies have landed (their mbarriers
        // completed), so the slot can be handed back with a plain store
        if (RING && tid == kOutThread) st_relaxed_gpu(done_flag(ring, h), static_cast<int>(gc0 + c + 1));

        // ---- MMA2a: S^T += delta^T Kb (thread 0);  MMA2b: Z_k^T += delta^T P^T,
        // O of chunk c (kOutThread, so that neither issuing thread is held up
        // by both; P of the next chunk is copied in once MMA2b is done)
        if (tid == 0) {
            tc_fence_after();
            const uint64_t da = tdesc(sb, S_DT), db = sdesc_mn32(sb + S_KB, IMG_BLK);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_tf32_ss(tmem + TS_S, kstep(da, 16384, s), mn_kstep(db, s), ID_N128_BMN, 1);
            mma_commit(bar_mma);
        } else if (tid == kOutThread) {
            tc_fence_after();
            const uint64_t da = tdesc(sb, S_DT), dp = tdesc(sb, S_P);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_tf32_ss(tmem + zcol(c), kstep(da, 16384, s), kstep(dp, IMG_BLK, s), ID_N64, 1);
            mma_commit(bar_o);
        }
        mma_pending = true;
        o_pending = true;
        t_prev = t0;
        if (c + 1 == nch) {   // last chunk: O straight to o once MMA2b is done
            if (!(ok = wait_all(bar_mma, mma_phase))) break;
            mma_phase ^= 1;   // the next sequence's products continue the phase count
            mma_pending = false;
            if (!(ok = wait_all(bar_o, (base + c) & 1))) break;
            o_pending = false;
            tc_fence_after();
            float acc[32];
            tmem_ld32(tm_lane(tmem, quarter, zcol(c) + 32 * half), acc);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int r = 32 * half + j;
                if (r < L) o[((size_t)(t0 + r) * H + h) * kD + e] = acc[j];
            }
        }
    }
    if (!ok) break;
    if (sT) {
        float acc[32];
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            const int c0 = 64 * half + 32 * part;
            tmem_ld32(tm_lane(tmem, quarter, TS_S + c0), acc);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) sT[state_off + (size_t)(c0 + j) * kD + e] = acc[j];
        }
    }
    base += static_cast<uint32_t>(nch);
    }   // sequences
    if (!ok && tid == 0) {
        // a bounded wait gave up: report, give outstanding copies and MMAs a
        // last bounded chance to land, then release tensor memory
        set_error(err, 2u);
        if (b1_pending) mbar_wait_bounded(bar_b1, b1_chunk & 1, 1u << 16);
        if (b2_pending) mbar_wait_bounded(bar_b2, b2_chunk & 1, 1u << 16);
        if (mma_pending) mbar_wait_bounded(bar_mma, mma_phase, 1u << 16);
        if (o_pending) mbar_wait_bounded(bar_o, 0, 1u << 16), mbar_wait_bounded(bar_o, 1, 1u << 16);
    }
    if (tid == kOutThread) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TS_COLS);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
kda_chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                      const float* __restrict__ g,
                      const float* __restrict__ beta, const int32_t* __restrict__ cu,
                      const int32_t* __restrict__ chunk_off, int N, int H, int64_t max_total, float scale,
                      int l2norm, int scalar_g, uint8_t* __restrict__ img, uint32_t* err) {
    prep_role<false>(&tm_q, &tm_k, &tm_v, &tm_g, g, beta, cu, chunk_off, N, H, max_total, scale, l2norm, scalar_g, img,
                     err, blockIdx.x, gridDim.x, Ring{nullptr, nullptr});
}

__global__ void __launch_bounds__(kThreads, 1)
kda_chunk_state_kernel(const __grid_constant__ CUtensorMap tm_o, const uint8_t* __restrict__ img,
                       const int32_t* __restrict__ chunk_off, const int32_t* __restrict__ cu, int64_t total_T, int H,
                       int64_t max_total, const float* s0, float* sT, float* __restrict__ o, uint32_t* err,
                       const int32_t* __restrict__ slots, int num_slots) {
    state_role<false>(&tm_o, img, chunk_off, cu, total_T, H, max_total, s0, sT, o, err, slots, num_slots,
                      blockIdx.x / H, blockIdx.x / H + 1, blockIdx.x % H, Ring{nullptr, nullptr});
}

// Both passes in one cooperative launch (all CTAs resident): CTAs 0 .. H-1
// carry the states of the H heads -- CTA h walks (sequence 0, head h),
// (sequence 1, head h), ... in order, so every head has the same amount of
// work -- and the others prepare chunks ahead of them through the ring, in
// the global chunk order (chunk-major over heads).  A head's ring slot and
// flags follow the global chunk index, which runs on across sequences.
__global__ void __launch_bounds__(kThreads, 1)
kda_chunk_overlap_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                         const __grid_constant__ CUtensorMap tm_o,
                         const float* __restrict__ g, const float* __restrict__ beta, const int32_t* __restrict__ cu,
                         const int32_t* __restrict__ chunk_off, int N, int H, int64_t total_T, int64_t max_total,
                         float scale, int l2norm, int scalar_g, uint8_t* __restrict__ img, const float* s0,
                         float* sT, float* __restrict__ o, uint32_t* err, const int32_t* __restrict__ slots,
                         int num_slots, Ring ring) {
    if (static_cast<int>(blockIdx.x) < H)
        state_role<true>(&tm_o, img, chunk_off, cu, total_T, H, max_total, s0, sT, o, err, slots, num_slots, 0, N,
                         blockIdx.x, ring);
    else
        prep_role<true>(&tm_q, &tm_k, &tm_v, &tm_g, g, beta, cu, chunk_off, N, H, max_total, scale, l2norm, scalar_g,
                        img, err, blockIdx.x - H, gridDim.x - H, ring);
}

int num_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 148;
}

size_t max_chunks(int32_t N, int64_t total_T) { return static_cast<size_t>((total_T + 63 * (int64_t)N) / kC); }
size_t index_bytes(int32_t N) { return (static_cast<size_t>(N + 1) * 4 + 1023) & ~size_t(1023); }

// Overlapped mode: at most 96 heads (one state CTA each, with enough SMs left
// for the prep role), any number of sequences.
constexpr int kMinPrepCtas = 16;
constexpr int kMaxRingHeads = 96;
bool ring_eligible(int32_t N, int32_t H) { return N >= 1 && H <= kMaxRingHeads; }
size_t ring_flag_bytes(int32_t H) { return (static_cast<size_t>(H) * 2 * kFlagStride * 4 + 1023) & ~size_t(1023); }

template <class K>
cudaError_t set_smem(K kernel, uint32_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

}  // namespace

size_t two_pass_scratch_bytes(int32_t N, int64_t total_T, int32_t H) {
    if (N < 0 || total_T < 0 || H <= 0) return 0;
    if (ring_eligible(N, H))
        return index_bytes(N) + ring_flag_bytes(H) + static_cast<size_t>(H) * kRing * IMG_BYTES;
    return index_bytes(N) + max_chunks(N, total_T) * static_cast<size_t>(H) * IMG_BYTES;
}

cudaError_t launch_chunk_two_pass(const PrefillArgs& a, void* scratch, cudaStream_t stream) {
    if (a.N == 0 || a.H == 0) return cudaSuccess;
    if (a.total_T <= 0) return cudaErrorInvalidValue;   // callers route empty batches elsewhere
    constexpr uint32_t O_SMEM = P_SMEM > S_SMEM ? P_SMEM : S_SMEM;
    static PerDeviceOnce attr_once;
    const cudaError_t attr_err = attr_once.run([] {
        cudaError_t e = set_smem(kda_chunk_prep_kernel, P_SMEM);
        if (e == cudaSuccess) e = set_smem(kda_chunk_state_kernel, S_SMEM);
        if (e == cudaSuccess) e = set_smem(kda_chunk_overlap_kernel, O_SMEM);
        return e;
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap mq, mk, mv, mg, mo;
    if (!make_token_map(&mq, a.q, a.total_T, a.H) || !make_token_map(&mk, a.k, a.total_T, a.H) ||
        !make_token_map(&mv, a.v, a.total_T, a.H) || !make_token_map(&mo, a.o, a.total_T, a.H, true))
        return cudaErrorInvalidValue;
    // g as [total_T, H, 128] fp32 for L2 prefetches (the scalar-decay form is not prefetched)
    if (a.scalar_decay) mg = mo;
    else if (!make_token_map(&mg, a.g, a.total_T, a.H, true)) return cudaErrorInvalidValue;
    int32_t* chunk_off = static_cast<int32_t*>(scratch);
    const int64_t max_total = static_cast<int64_t>(max_chunks(a.N, a.total_T));
    const int sms = num_sms();

    if (ring_eligible(a.N, a.H)) {
        // both passes in one cooperative launch: H state CTAs + the rest preparing
        int dev = 0, coop = 0, per_sm = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kda_chunk_overlap_kernel, kThreads, O_SMEM) !=
                cudaSuccess)
            return cudaErrorUnknown;
        if (!coop || per_sm < 1 || a.H + kMinPrepCtas > sms) return cudaErrorNotSupported;
        uint8_t* flags = static_cast<uint8_t*>(scratch) + index_bytes(a.N);
        Ring ring{reinterpret_cast<int32_t*>(flags), reinterpret_cast<int32_t*>(flags) + a.H * kFlagStride};
        uint8_t* img = flags + ring_flag_bytes(a.H);
        cudaError_t e = launch_kernel(kda_chunk_index_kernel, dim3(1), dim3(1024), 0, stream, a.cu_seqlens, a.N,
                                      a.total_T, max_total, chunk_off, a.err, ring.ready, a.H * 2 * kFlagStride);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(sms));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = O_SMEM;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(
            &cfg, kda_chunk_overlap_kernel, mq, mk, mv, mg, mo, a.g, a.beta, a.cu_seqlens,
            static_cast<const int32_t*>(chunk_off), static_cast<int>(a.N), static_cast<int>(a.H), a.total_T,
            max_total, a.scale,
            a.l2norm ? 1 : 0, a.scalar_decay ? 1 : 0, img, a.initial_state, a.final_state, a.o, a.err, a.slots,
            static_cast<int>(a.num_slots), ring);
        return e;
    }

    uint8_t* img = static_cast<uint8_t*>(scratch) + index_bytes(a.N);
    cudaError_t e = launch_kernel(kda_chunk_index_kernel, dim3(1), dim3(1024), 0, stream, a.cu_seqlens, a.N,
                                  a.total_T, max_total, chunk_off, a.err, static_cast<int32_t*>(nullptr), 0);
    if (e != cudaSuccess) return e;
    const size_t items_ub = max_chunks(a.N, a.total_T) * static_cast<size_t>(a.H);
    const size_t grid1 = items_ub < static_cast<size_t>(sms) ? items_ub : static_cast<size_t>(sms);
    if (grid1 > 0) {
        e = launch_kernel(kda_chunk_prep_kernel, dim3(static_cast<unsigned>(grid1)), dim3(kThreads), P_SMEM, stream,
                          mq, mk, mv, mg, a.g, a.beta, a.cu_seqlens, static_cast<const int32_t*>(chunk_off), a.N, a.H,
                          max_total, a.scale, a.l2norm ? 1 : 0, a.scalar_decay ? 1 : 0, img, a.err);
        if (e != cudaSuccess) return e;
    }
    const long long blocks = (long long)a.N * a.H;
    return launch_kernel(kda_chunk_state_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), S_SMEM, stream,
                         mo, static_cast<const uint8_t*>(img), static_cast<const int32_t*>(chunk_off), a.cu_seqlens,
                         a.total_T, a.H, max_total, a.initial_state, a.final_state, a.o, a.err, a.slots,
                         static_cast<int>(a.num_slots));
}

}  // namespace kda
