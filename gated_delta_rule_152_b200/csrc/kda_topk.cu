// kda_topk.cu -- the selection step of the lightning indexer: per query row,
// the k best of n per-token scores (page "GLM-5.3-FLASH", dimsnsums.com,
// section "How can a layer search the whole history selectively?": the
// indexer of a sparse layer scores all earlier tokens and passes only the
// best 2,048 on to full attention).
//
// Order of tokens: a higher score ranks higher; equal scores (-0 == +0) rank
// the lower index higher, so the kept set is unique.  The output lists the
// kept indices best first; -1 fills the slots past n when n < k.
//
// Scores become 32-bit keys whose unsigned order is the float order (sign
// bit set for positives, all bits inverted for negatives), and the cut is
// found by radix selection on the keys, most significant digit first:
//   1. hist0 (many CTAs per row): histogram of the top 11 key bits;
//   2. pick0 (one CTA per row): the top-digit bin b holding the k-th best key;
//   3. split (many CTAs per row): the keys of bin b and above become candidates
//      (when bin b holds at most kTopkCap keys);
//   4. finish (one CTA per row): the remaining digits (and, for equal keys at
//      the cut, the index digits) among the candidates -- or over the whole
//      row when bin b holds more than kTopkCap keys -- then a bitonic sort of
//      the k kept (key, index) pairs, best first.
// HBM traffic in the common case: the scores are read twice (steps 1 and 3).
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/kda.h"
#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kBins = 2048;               // 11-bit digits
constexpr int kSeg = 16384;               // scores per CTA in the row-parallel passes
constexpr int kTopkMaxK = 4096;
constexpr int kTopkCap = 16384;           // candidates kept per row for the finish step
constexpr int kCandCap = kTopkCap + kTopkMaxK;   // candidates: bin b and the keys above it
constexpr int kSplitStage = 1024;         // pairs one split CTA stages in shared memory

struct RowState {
    int32_t n;        // tokens in the row
    int32_t need;     // keys still to take from bin b
    uint32_t b;       // top-digit bin of the cut
    int32_t cnt_b;    // keys in bin b
    int32_t nsel;     // kept pairs written to the row's buffer
    int32_t ncand;    // candidates written (bin b and the keys above it)
    int32_t mode;     // 0: n <= k, keep all; 1: candidates; 2: bin b too full, the finish step scans the row
    int32_t pad[9];
};
static_assert(sizeof(RowState) == 64, "row state");

// Workspace (after the 256-byte header with the error word): per row its
// state, then [rows][kBins] histogram counts, [rows][k] kept pairs and
// [rows][kCandCap] candidates.
struct Layout {
    RowState* st;
    uint32_t* hist;
    unsigned long long* kept;
    unsigned long long* cand;
};
__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
__host__ __device__ inline Layout layout(void* ws, int rows, int k) {
    uint8_t* p = static_cast<uint8_t*>(ws) + 256;
    Layout l;
    l.st = reinterpret_cast<RowState*>(p);
    p += align256(sizeof(RowState) * static_cast<size_t>(rows));
    l.hist = reinterpret_cast<uint32_t*>(p);
    p += align256(sizeof(uint32_t) * kBins * static_cast<size_t>(rows));
    l.kept = reinterpret_cast<unsigned long long*>(p);
    p += align256(sizeof(unsigned long long) * static_cast<size_t>(k) * rows);
    l.cand = reinterpret_cast<unsigned long long*>(p);
    return l;
}
inline size_t workspace_bytes(int rows, int k) {
    return 256 + align256(sizeof(RowState) * static_cast<size_t>(rows)) +
           align256(sizeof(uint32_t) * kBins * static_cast<size_t>(rows)) +
           align256(sizeof(unsigned long long) * static_cast<size_t>(k) * rows) +
           sizeof(unsigned long long) * static_cast<size_t>(kCandCap) * rows;
}

// Order-preserving key of a score; -0 and +0 get the same key (the IEEE sum
// x + 0 turns -0 into +0 and leaves every other non-NaN score as it is).
// Positives get the sign bit set, negatives all bits inverted.
__device__ __forceinline__ uint32_t score_key(float x) {
    const uint32_t u = __float_as_uint(x + 0.0f);
    return u ^ (static_cast<uint32_t>(static_cast<int32_t>(u) >> 31) | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}
// A kept (key, index) pair as one 64-bit value whose unsigned order is the
// ranking: the key, then the lower index first.
__device__ __forceinline__ unsigned long long pair_of(uint32_t key, int32_t idx) {
    return (static_cast<unsigned long long>(key) << 32) | static_cast<uint32_t>(~idx);
}

__device__ __forceinline__ int row_len(const int32_t* lengths, int r, int64_t n) {
    if (!lengths) return static_cast<int>(n);
    const int64_t l = lengths[r];
    return static_cast<int>(l < 0 ? 0 : (l > n ? n : l));
}

// First index >= lo whose score sits on a 16-byte boundary (rows need only be
// 4-byte aligned, so the row stride may be any number of scores).
__device__ __forceinline__ int aligned_from(const float* row, int lo) {
    const int mis = static_cast<int>((reinterpret_cast<uintptr_t>(row + lo) >> 2) & 3u);
    return lo + ((4 - mis) & 3);
}

// Visit the scores [lo, hi) of one row as (index, key), 4 at a time where aligned.
template <class F>
__device__ __forceinline__ void for_keys(const float* row, int lo, int hi, int t, int nt, F f) {
    const int lo4 = aligned_from(row, lo), hi4 = lo4 + ((hi - lo4) & ~3);
    if (lo4 >= hi) {
        for (int i = lo + t; i < hi; i += nt) f(i, score_key(__ldg(row + i)));
        return;
    }
    for (int i = lo + t; i < lo4; i += nt) f(i, score_key(__ldg(row + i)));
#pragma unroll 4
    for (int i = lo4 + 4 * t; i < hi4; i += 4 * nt) {
        const float4 v = __ldcs(reinterpret_cast<const float4*>(row + i));
        f(i, score_key(v.x));
        f(i + 1, score_key(v.y));
        f(i + 2, score_key(v.z));
        f(i + 3, score_key(v.w));
    }
    for (int i = hi4 + t; i < hi; i += nt) f(i, score_key(__ldg(row + i)));
}

// Warp-aggregated append of (key, idx) to a buffer in shared memory.
__device__ __forceinline__ void append_shared(bool take, unsigned long long v, int* counter, unsigned long long* buf,
                                              int cap) {
    const unsigned m = __ballot_sync(0xffffffffu, take);
    if (!m) return;
    const int lane = threadIdx.x & 31, leader = __ffs(m) - 1;
    int base = 0;
    if (lane == leader) base = atomicAdd(counter, __popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (take) {
        const int pos = base + __popc(m & ((1u << lane) - 1u));
        if (pos < cap) buf[pos] = v;
    }
}
// The same append staged in shared memory: the pairs of one CTA collect in `sh`
// (cap_sh of them; any further ones go straight to the row's buffer), and
// flush_staged moves them out with one reservation on the row's counter.
__device__ __forceinline__ void append_staged(bool take, unsigned long long v, int* sh_count,
                                              unsigned long long* sh, int cap_sh, int32_t* counter,
                                              unsigned long long* buf, int cap) {
    const unsigned m = __ballot_sync(0xffffffffu, take);
    if (!m) return;
    const int lane = threadIdx.x & 31, leader = __ffs(m) - 1;
    int base = 0;
    if (lane == leader) base = atomicAdd(sh_count, __popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (take) {
        const int pos = base + __popc(m & ((1u << lane) - 1u));
        if (pos < cap_sh) {
            sh[pos] = v;
        } else {
            const int g = atomicAdd(counter, 1);
            if (g < cap) buf[g] = v;
        }
    }
}
// append_staged for four pairs per lane at once (one shared-memory reservation
// for the warp); all 32 lanes call it.
__device__ __forceinline__ void append4_staged(const bool (&take)[4], const unsigned long long (&v)[4], int* sh_count,
                                               unsigned long long* sh, int cap_sh, int32_t* counter,
                                               unsigned long long* buf, int cap) {
    unsigned m[4];
    int tot = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        m[j] = __ballot_sync(0xffffffffu, take[j]);
        tot += __popc(m[j]);
    }
    if (tot == 0) return;
    const int lane = threadIdx.x & 31;
    int base = 0;
    if (lane == 0) base = atomicAdd(sh_count, tot);
    base = __shfl_sync(0xffffffffu, base, 0);
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (take[j]) {
            const int pos = base + __popc(m[j] & lt);
            if (pos < cap_sh) {
                sh[pos] = v[j];
            } else {
                const int g = atomicAdd(counter, 1);
                if (g < cap) buf[g] = v[j];
            }
        }
        base += __popc(m[j]);
    }
}
// All threads; a block barrier first.
__device__ __forceinline__ void flush_staged(const int* sh_count, const unsigned long long* sh, int cap_sh,
                                             int32_t* counter, unsigned long long* buf, int cap, int* sh_base) {
    __syncthreads();
    const int n = min(*sh_count, cap_sh);
    if (threadIdx.x == 0 && n > 0) *sh_base = atomicAdd(counter, n);
    __syncthreads();
    if (n == 0) return;
    const int g0 = *sh_base;
    for (int i = threadIdx.x; i < n; i += blockDim.x)
        if (g0 + i < cap) buf[g0 + i] = sh[i];
}

__global__ void __launch_bounds__(kThreads) kda_topk_init_kernel(const int32_t* lengths, int64_t n, int k, Layout L) {
    const int r = blockIdx.x;
    if (threadIdx.x == 0) {
        RowState s = {};
        s.n = row_len(lengths, r, n);
        s.mode = s.n <= k ? 0 : 1;
        L.st[r] = s;
    }
    for (int i = threadIdx.x; i < kBins; i += kThreads) L.hist[static_cast<size_t>(r) * kBins + i] = 0u;
}

// Histogram of the top 11 key bits of one segment of one row (counts of each
// pair of warps in shared memory, then one global add per non-empty bin).
constexpr int kSubHists = kThreads / 64;
__global__ void __launch_bounds__(kThreads) kda_topk_hist0_kernel(const float* __restrict__ scores, int64_t ld,
                                                                  Layout L) {
    __shared__ uint32_t h[kSubHists][kBins];
    const int r = blockIdx.y;
    const RowState s = L.st[r];
    const int lo = blockIdx.x * kSeg, hi = min(s.n, lo + kSeg);
    if (s.mode == 0 || lo >= hi) return;
    const int sub = threadIdx.x >> 6;
    for (int i = threadIdx.x; i < kSubHists * kBins; i += kThreads) (&h[0][0])[i] = 0u;
    __syncthreads();
    for_keys(scores + r * ld, lo, hi, threadIdx.x, kThreads,
             [&](int, uint32_t key) { atomicAdd(&h[sub][key >> 21], 1u); });
    __syncthreads();
    for (int b = threadIdx.x; b < kBins; b += kThreads) {
        uint32_t c = 0;
#pragma unroll
        for (int w = 0; w < kSubHists; ++w) c += h[w][b];
        if (c) atomicAdd(&L.hist[static_cast<size_t>(r) * kBins + b], c);
    }
}

// Block-wide search over a 2048-bin histogram `h` (shared memory) for the bin
// that holds the `need`-th element counted from the top (from_top) or from
// the bottom.  Returns the bin; *before receives the count of the bins
// passed over first.  All threads call it; two block barriers inside.
template <int NT>
__device__ __forceinline__ int find_bin(const uint32_t* h, int need, bool from_top, int* before, int* scratch) {
    static_assert(NT % 32 == 0 && NT <= 1024 && kBins % NT == 0, "find_bin: whole warps, at most 32");
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    constexpr int per = kBins / NT;   // bins per thread, thread 0 first in visiting order
    if (t == 0) scratch[32] = scratch[33] = 0;
    uint32_t c[per], sum = 0;
#pragma unroll
    for (int j = 0; j < per; ++j) {
        const int b = from_top ? kBins - 1 - (per * t + j) : per * t + j;
        c[j] = h[b];
        sum += c[j];
    }
    // exclusive scan of the per-thread sums in visiting order
    uint32_t x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = static_cast<int>(x);
    __syncthreads();
    uint32_t woff = 0;
    for (int w = 0; w < warp; ++w) woff += static_cast<uint32_t>(scratch[w]);
    uint32_t run = woff + x - sum;
    if (run < static_cast<uint32_t>(need) && run + sum >= static_cast<uint32_t>(need)) {
#pragma unroll
        for (int j = 0; j < per; ++j) {
            if (run + c[j] >= static_cast<uint32_t>(need)) {
                scratch[32] = from_top ? kBins - 1 - (per * t + j) : per * t + j;
                scratch[33] = static_cast<int>(run);
                break;
            }
            run += c[j];
        }
    }
    __syncthreads();
    *before = scratch[33];
    return scratch[32];
}

__global__ void __launch_bounds__(kThreads) kda_topk_pick0_kernel(int k, Layout L) {
    __shared__ uint32_t h[kBins];
    __shared__ int scratch[40];
    const int r = blockIdx.x;
    RowState s = L.st[r];
    if (s.mode == 0) return;
    for (int i = threadIdx.x; i < kBins; i += kThreads) h[i] = L.hist[static_cast<size_t>(r) * kBins + i];
    __syncthreads();
    int above = 0;
    const int b = find_bin<kThreads>(h, k, true, &above, scratch);
    if (threadIdx.x == 0) {
        s.b = static_cast<uint32_t>(b);
        s.need = k - above;
        s.cnt_b = static_cast<int>(h[b]);
        s.mode = s.cnt_b <= kTopkCap ? 1 : 2;
        L.st[r] = s;
    }
}

// Keys in bin b or above are candidates (mode 1); every key is kept when the
// row has at most k tokens (mode 0).
__global__ void __launch_bounds__(kThreads) kda_topk_split_kernel(const float* __restrict__ scores, int64_t ld,
                                                                  int k, Layout L) {
    const int r = blockIdx.y;
    RowState* sp = L.st + r;
    const RowState s = *sp;
    const int lo = blockIdx.x * kSeg, hi = min(s.n, lo + kSeg);
    if (s.mode == 2) return;
    // mode 0: every pair to the kept buffer; mode 1: the candidates
    unsigned long long* buf =
        s.mode == 0 ? L.kept + static_cast<size_t>(r) * k : L.cand + static_cast<size_t>(r) * kCandCap;
    int32_t* counter = s.mode == 0 ? &sp->nsel : &sp->ncand;
    const int cap = s.mode == 0 ? k : kCandCap;
    // whole warps iterate together so that the warp-wide append sees every lane;
    // four scores per thread and step between 16-byte boundaries
    const float* row = scores + r * ld;
    // this CTA's pairs, staged in shared memory
    __shared__ unsigned long long sh_buf[kSplitStage];
    __shared__ int sh_n, sh_base;
    auto visit = [&](int i, uint32_t key, bool live) {
        append_staged(live && (s.mode == 0 || (key >> 21) >= s.b), pair_of(key, i), &sh_n, sh_buf, kSplitStage,
                      counter, buf, cap);
    };
    if (hi <= lo) return;
    if (threadIdx.x == 0) sh_n = 0;
    __syncthreads();
    const int lo4 = min(aligned_from(row, lo), hi), hi4 = lo4 + ((hi - lo4) & ~3);
    if (threadIdx.x < 32) {   // up to three scores before the first 16-byte boundary: one warp
        const int i = lo + static_cast<int>(threadIdx.x);
        const bool live = i < lo4;
        visit(i, live ? score_key(row[i]) : 0u, live);
    }
    // The filter below needs no keys when bin b's lowest key is that of a number fb:
    // key(x) >= b << 21 exactly when x >= fb (the key order is the float order, -0
    // and +0 alike); bins 0-3 and 2044-2047 begin among the NaN bit patterns
    const bool by_float = s.mode == 1 && s.b >= 4u && s.b < 2044u;
    const float fb = by_float ? key_score(s.b << 21) : 0.f;
    for (int base = lo4; base < hi4; base += 4 * kThreads) {
        const int i = base + 4 * static_cast<int>(threadIdx.x);
        const bool live = i < hi4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (live) v = __ldcs(reinterpret_cast<const float4*>(row + i));
        // most steps keep nothing: a warp whose scores all lie below bin b skips the appends
        bool maybe;
        if (by_float) {
            maybe = live && fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)) >= fb;
        } else {
            const uint32_t top = max(max(score_key(v.x), score_key(v.y)), max(score_key(v.z), score_key(v.w))) >> 21;
            maybe = live && (s.mode == 0 || top >= s.b);
        }
        if (!__any_sync(0xffffffffu, maybe)) continue;
        const uint32_t k0 = score_key(v.x), k1 = score_key(v.y), k2 = score_key(v.z), k3 = score_key(v.w);
        const bool take[4] = {live && (s.mode == 0 || (k0 >> 21) >= s.b), live && (s.mode == 0 || (k1 >> 21) >= s.b),
                              live && (s.mode == 0 || (k2 >> 21) >= s.b), live && (s.mode == 0 || (k3 >> 21) >= s.b)};
        const unsigned long long pv[4] = {pair_of(k0, i), pair_of(k1, i + 1), pair_of(k2, i + 2), pair_of(k3, i + 3)};
        append4_staged(take, pv, &sh_n, sh_buf, kSplitStage, counter, buf, cap);
    }
    if (threadIdx.x < 32) {   // up to three scores after the last boundary: one warp
        const int i = hi4 + static_cast<int>(threadIdx.x);
        const bool live = i < hi;
        visit(i, live ? score_key(row[i]) : 0u, live);
    }
    flush_staged(&sh_n, sh_buf, kSplitStage, counter, buf, cap, &sh_base);
}

// One compare-exchange stage in registers: stride s (< 64) of block size `size`.
__device__ __forceinline__ void bitonic_reg_stage(ulonglong2& x, int v, int size, int s) {
    const bool desc = ((2 * v) & size) == 0;
    if (s == 1) {
        if ((x.x < x.y) == desc) {
            const unsigned long long tmp = x.x;
            x.x = x.y;
            x.y = tmp;
        }
    } else {
        const int hs = s >> 1;
        const unsigned long long y0 = __shfl_xor_sync(0xffffffffu, x.x, hs);
        const unsigned long long y1 = __shfl_xor_sync(0xffffffffu, x.y, hs);
        const bool keep_max = ((v & hs) == 0) == desc;   // the lower thread holds the lower index
        x.x = keep_max ? (x.x > y0 ? x.x : y0) : (x.x < y0 ? x.x : y0);
        x.y = keep_max ? (x.y > y1 ? x.y : y1) : (x.y < y1 ? x.y : y1);
    }
}

// Bitonic sort, descending, of the P pairs in a (P a power of two, P <= 4 NT),
// by all NT threads; ends with a block barrier.  Strides of 64 and more take
// a shared-memory pass and a block barrier each; the strides below 64 of every
// merge run in registers, elements 2v and 2v+1 in (virtual) thread v, with the
// partner element of stride s >= 2 in thread v ^ (s / 2) of the same warp.
// Descending runs (the compare direction of block `size` containing the pair)
// build the final descending order.
template <int NT>
__device__ __forceinline__ void bitonic_desc(unsigned long long* a, int P) {
    const int t = threadIdx.x, nv = P >> 1;
    // whole warps over the virtual threads (for the shuffles); lanes past nv carry zeros
    auto each_warp = [&](auto body) {
        for (int v0 = t & ~31; v0 < nv; v0 += NT) {
            const int v = v0 + (t & 31);
            const bool live = v < nv;
            ulonglong2 x = live ? *reinterpret_cast<const ulonglong2*>(a + 2 * v) : make_ulonglong2(0ull, 0ull);
            body(x, v);
            if (live) *reinterpret_cast<ulonglong2*>(a + 2 * v) = x;
        }
    };
    if (P >= 64) {
        each_warp([&](ulonglong2& x, int v) {
#pragma unroll
            for (int size = 2; size <= 64; size <<= 1)
#pragma unroll
                for (int st = size >> 1; st >= 1; st >>= 1) bitonic_reg_stage(x, v, size, st);
        });
    } else if (P >= 2) {
        each_warp([&](ulonglong2& x, int v) {
            for (int size = 2; size <= P; size <<= 1)
                for (int st = size >> 1; st >= 1; st >>= 1) bitonic_reg_stage(x, v, size, st);
        });
    }
    __syncthreads();
    for (int size = 128; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride >= 64; stride >>= 1) {
            for (int i = t; i < nv; i += NT) {
                const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const unsigned long long x = a[lo], y = a[hi];
                if ((x < y) == desc) {
                    a[lo] = y;
                    a[hi] = x;
                }
            }
            __syncthreads();
        }
        each_warp([&](ulonglong2& x, int v) {
#pragma unroll
            for (int st = 32; st >= 1; st >>= 1) bitonic_reg_stage(x, v, size, st);
        });
        __syncthreads();
    }
}

// One CTA per row: the rest of the cut, the kept set, and the sorted output.
constexpr int kFinishThreads = 1024;
__global__ void __launch_bounds__(kFinishThreads) kda_topk_finish_kernel(const float* __restrict__ scores, int64_t ld,
                                                                         int k, Layout L, int32_t* __restrict__ out_idx,
                                                                         float* __restrict__ out_val) {
    constexpr int NT = kFinishThreads;
    __shared__ uint32_t h[kBins];
    __shared__ int scratch[40];
    __shared__ __align__(16) unsigned long long sorted[kTopkMaxK];
    __shared__ int sh_nsel;   // kept pairs gathered into `sorted`
    const int r = blockIdx.x, t = threadIdx.x;
    if (t == 0) sh_nsel = 0;
    RowState* sp = L.st + r;
    const RowState s = *sp;
    unsigned long long* kept = L.kept + static_cast<size_t>(r) * k;
    const unsigned long long* cand = L.cand + static_cast<size_t>(r) * kCandCap;
    const int ncand = s.ncand < kCandCap ? s.ncand : kCandCap;
    const float* row = scores + r * ld;

    if (s.mode != 0) {
        // the source of the remaining selection: the candidates (mode 1) or the whole row (mode 2);
        // visit(f) calls f(key, idx) for every key of bin b (the caller filters further)
        auto visit = [&](auto f) {
            if (s.mode == 1) {
                for (int i = t; i < ncand; i += NT) {
                    const unsigned long long v = cand[i];
                    f(static_cast<uint32_t>(v >> 32), static_cast<int32_t>(~static_cast<uint32_t>(v)));
                }
            } else {
                for_keys(row, 0, s.n, t, NT, [&](int i, uint32_t key) {
                    if ((key >> 21) == s.b) f(key, i);
                });
            }
        };
        // remaining key digits: bits 20..10, then 9..0
        uint32_t prefix = s.b << 21, mask = 0xFFE00000u;
        int need = s.need, eq_total = 0;
        for (int pass = 0; pass < 2; ++pass) {
            const int shift = pass == 0 ? 10 : 0;
            const uint32_t dmask = pass == 0 ? 0x7FFu : 0x3FFu;
            for (int i = t; i < kBins; i += NT) h[i] = 0u;
            __syncthreads();
            visit([&](uint32_t key, int32_t) {
                if ((key & mask) == prefix) atomicAdd(&h[(key >> shift) & dmask], 1u);
            });
            __syncthreads();
            int above = 0;
            const int bin = find_bin<NT>(h, need, true, &above, scratch);
            prefix |= static_cast<uint32_t>(bin) << shift;
            mask |= dmask << shift;
            need -= above;
            eq_total = static_cast<int>(h[bin]);
            __syncthreads();
        }
        const uint32_t T = prefix;   // the key at the cut; `need` of the eq_total keys equal to it are kept
        // ties at the cut: the need-th smallest index among the keys equal to T (index bits 30..20, 19..10, 9..0)
        int32_t last = 0x7FFFFFFF;
        if (need < eq_total) {
            uint32_t ip = 0, im = 0;
            for (int pass = 0; pass < 3; ++pass) {
                const int shift = pass == 0 ? 20 : (pass == 1 ? 10 : 0);
                const uint32_t dmask = pass == 0 ? 0x7FFu : 0x3FFu;
                for (int i = t; i < kBins; i += NT) h[i] = 0u;
                __syncthreads();
                visit([&](uint32_t key, int32_t idx) {
                    const uint32_t u = static_cast<uint32_t>(idx);
                    if (key == T && (u & im) == ip) atomicAdd(&h[(u >> shift) & dmask], 1u);
                });
                __syncthreads();
                int below = 0;
                const int bin = find_bin<NT>(h, need, false, &below, scratch);
                ip |= static_cast<uint32_t>(bin) << shift;
                im |= dmask << shift;
                need -= below;
                __syncthreads();
            }
            last = static_cast<int32_t>(ip);
        }
        // keep the keys above the cut and the equal keys up to index `last`
        // (whole warps iterate together for the warp-wide append)
        if (s.mode == 1) {
            for (int base = 0; base < ncand; base += NT) {
                const int i = base + t;
                unsigned long long v = 0;
                bool take = false;
                if (i < ncand) {
                    v = cand[i];
                    const uint32_t key = static_cast<uint32_t>(v >> 32);
                    const int32_t idx = static_cast<int32_t>(~static_cast<uint32_t>(v));
                    take = key > T || (key == T && idx <= last);
                }
                append_shared(take, v, &sh_nsel, sorted, kTopkMaxK);
            }
        } else {
            for (int base = 0; base < s.n; base += NT) {
                const int i = base + t;
                bool take = false;
                unsigned long long v = 0;
                if (i < s.n) {
                    const uint32_t key = score_key(row[i]);
                    v = pair_of(key, i);
                    take = key > T || (key == T && i <= last);
                }
                append_shared(take, v, &sh_nsel, sorted, kTopkMaxK);
            }
        }
        __syncthreads();
    }
    // bitonic sort, best first, of the m kept pairs (padded with zeros, which rank last):
    // gathered into `sorted` above, or written by the split step when the row has at
    // most k tokens
    const int m = s.n < k ? s.n : k;
    int P = 1;
    while (P < m) P <<= 1;
    if (s.mode == 0) {
        for (int i = t; i < P; i += NT) sorted[i] = i < m ? kept[i] : 0ull;
    } else {
        for (int i = m + t; i < P; i += NT) sorted[i] = 0ull;
    }
    __syncthreads();
    bitonic_desc<NT>(sorted, P);
    for (int i = t; i < k; i += NT) {
        const bool live = i < m;
        const unsigned long long v = live ? sorted[i] : 0ull;
        out_idx[static_cast<size_t>(r) * k + i] = live ? static_cast<int32_t>(~static_cast<uint32_t>(v)) : -1;
        if (out_val)
            out_val[static_cast<size_t>(r) * k + i] = live ? key_score(static_cast<uint32_t>(v >> 32)) : -INFINITY;
    }
}

}  // namespace
}  // namespace kda

extern "C" {

size_t kda_topk_workspace_size(int32_t rows, int64_t n, int32_t k) {
    if (rows < 0 || n < 0 || n >= (int64_t(1) << 31) || k < 1 || k > kda::kTopkMaxK) return 0;
    return kda::workspace_bytes(rows, k);
}

int kda_topk_indices(const float* scores, int64_t ld, int32_t rows, int64_t n, int32_t k,
                     const int32_t* row_lengths, int32_t* indices, float* values, void* workspace,
                     size_t workspace_bytes, kda_stream_t stream) {
    using namespace kda;
    if (rows < 0 || n < 0 || n >= (int64_t(1) << 31) || ld < n || rows > 65535) return KDA_ERR_INVALID_ARG;
    if (k < 1 || k > kTopkMaxK) return KDA_ERR_UNSUPPORTED;
    if (rows == 0) return KDA_OK;
    if (!indices || (n > 0 && !scores)) return KDA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(scores) & 3u) || (reinterpret_cast<uintptr_t>(indices) & 3u) ||
        (reinterpret_cast<uintptr_t>(values) & 3u) || (reinterpret_cast<uintptr_t>(row_lengths) & 3u))
        return KDA_ERR_MISALIGNED;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < kda_topk_workspace_size(rows, n, k))
        return KDA_ERR_WORKSPACE;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (major != 10) return KDA_ERR_UNSUPPORTED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Layout L = layout(workspace, rows, k);
    const unsigned segs = static_cast<unsigned>((n + kSeg - 1) / kSeg > 0 ? (n + kSeg - 1) / kSeg : 1);
    const dim3 grid2(segs, static_cast<unsigned>(rows));
    cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(uint32_t), s);
    if (e == cudaSuccess) e = launch_kernel(kda_topk_init_kernel, dim3(rows), dim3(kThreads), 0, s, row_lengths, n, k, L);
    if (e == cudaSuccess) e = launch_kernel(kda_topk_hist0_kernel, grid2, dim3(kThreads), 0, s, scores, ld, L);
    if (e == cudaSuccess) e = launch_kernel(kda_topk_pick0_kernel, dim3(rows), dim3(kThreads), 0, s, k, L);
    if (e == cudaSuccess) e = launch_kernel(kda_topk_split_kernel, grid2, dim3(kThreads), 0, s, scores, ld, k, L);
    if (e == cudaSuccess)
        e = launch_kernel(kda_topk_finish_kernel, dim3(rows), dim3(kFinishThreads), 0, s, scores, ld, k, L, indices,
                          values);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
