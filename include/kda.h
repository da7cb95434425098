/*
 * kda.h -- C ABI of the Kimi Delta Attention (KDA) layer core for NVIDIA B200
 * (sm_100a).  Library: gated_delta_rule_152_b200/libkda.so.
 *
 * The operation (page "GLM-5.3-FLASH", dimsnsums.com/models/glm-5-3-flash/
 * attention, section "How can a layer remember without rereading?", the
 * displayed update rule): every (sequence, head) carries a d x d state S
 * (d = 128, rows = key channels, columns = value channels) updated per token as
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *
 * with a per-channel decay alpha_t = exp(g_t) in (0,1]^d and write strength
 * beta_t, and emits o_t = scale * S_t^T q_t from the updated state.  With
 * KDA_FLAG_L2NORM_QK, q_t and k_t are first divided by sqrt(sum(x^2) + 1e-6)
 * over the head's d channels.  Sequences and heads are independent.
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates and frees nothing.  Every pointer must be 16-byte aligned.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous: a KDA_OK return means the launch was
 *     accepted, not that the kernel finished.
 *   - Layouts are row-major and contiguous:
 *       q, k, v, g : [tokens, H, d]      (token, head, channel)
 *       beta       : [tokens, H]
 *       o          : [tokens, H, d]      fp32
 *       states     : [N, H, d, d] fp32   (sequence, head, key row, value col)
 *   - q, k, v share one dtype (kda_dtype); g, beta, states and o are fp32.
 *   - g = log(alpha) must be finite and <= 0; any such value is handled
 *     exactly (up to rounding) by every path.  The page lets each channel
 *     decay at its own data-dependent rate, so a chunk may carry any amount
 *     of decay: the chunked tensor-core prefill takes a 64-token chunk whose
 *     decay exceeds about 69 nats in some channel through 16-token block
 *     references, and pairs of tokens inside a 16-token block whose decay
 *     exceeds that through one exponential each (both slower than the common
 *     case, still exact); the fused kernel that runs with the minimum
 *     workspace hands such a sequence to the token-by-token recurrence.
 *   - Only d == 128 is supported (KDA_ERR_UNSUPPORTED otherwise).
 *   - Returns KDA_OK (0) or a negative kda_status.  Host-side checks run
 *     before anything is enqueued; on an error nothing is launched.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kda_stream_t; /* same type as cudaStream_t */

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = -1, /* NULL required pointer, negative size, bad cu_seqlens length */
    KDA_ERR_UNSUPPORTED = -2, /* d != 128, unsupported dtype or flag, device not sm_100 */
    KDA_ERR_MISALIGNED = -3,  /* a pointer is not 16-byte aligned */
    KDA_ERR_WORKSPACE = -4,   /* workspace NULL or smaller than kda_chunk_fwd_workspace_size_min() */
    KDA_ERR_CUDA = -5         /* a CUDA runtime call or kernel launch failed */
} kda_status;

typedef enum { KDA_DTYPE_BF16 = 0, KDA_DTYPE_FP32 = 1 } kda_dtype;

enum {
    /* L2-normalise q and k per token and head inside the kernel. */
    KDA_FLAG_L2NORM_QK = 1u,
    /* Force the token-by-token fp32 kernel for prefill (default for FP32
     * inputs; for BF16 inputs the chunked tensor-core kernel is the default). */
    KDA_FLAG_RECURRENT = 2u,
    /* Gated-DeltaNet form: one decay per (token, head) shared by all d
     * channels, Diag(alpha_t) = alpha_t I.  g is then [tokens, H] instead of
     * [tokens, H, d] (decode: [N, H]).  The page names this scalar-gated
     * delta rule (GDN) as the baseline KDA refines; it is KDA with equal
     * per-channel decays, and every kernel accepts it. */
    KDA_FLAG_SCALAR_DECAY = 4u
};

/* Device-side error bits, OR-ed into the first 32-bit word of the workspace by
 * kda_chunk_fwd and readable with kda_workspace_error(). */
enum {
    KDA_DEVERR_CU_SEQLENS = 1u, /* cu_seqlens not non-decreasing in [0, total_T]; the
                                   offending sequences were treated as empty */
    KDA_DEVERR_TIMEOUT = 2u,    /* a bounded wait inside a kernel gave up; outputs of the
                                   affected (sequence, head) are undefined */
    KDA_DEVERR_SLOT = 4u        /* kda_chunk_fwd_slots: a slot index outside [0, num_slots);
                                   that sequence was skipped */
};

/*
 * Bytes of device workspace with which kda_chunk_fwd (and _slots) runs its
 * fastest path for these sizes: the error word, a chunk index, and room for
 * the state-independent tensor-core operands of the (64-token chunk, head)
 * pairs, 145 KiB per pair.  With at most 96 heads that is a ring of 8 such
 * slots per head plus one 128-byte flag line per head and direction,
 * whatever the number and lengths of the sequences (32 heads: about 38 MB);
 * with more heads every pair has its own slot (2 x 8192 tokens x 100 heads:
 * about 1.9 GB).  Returns 0 for invalid sizes.
 */
KDA_API size_t kda_chunk_fwd_workspace_size(int32_t N, int64_t total_T, int32_t H, int32_t d,
                                    kda_dtype dt);

/*
 * The smallest workspace the prefill calls accept: the error word plus 4
 * bytes per sequence.  With less than kda_chunk_fwd_workspace_size() the
 * bf16 prefill runs a single fused kernel per (sequence, head, 32-column
 * value slice) instead of the two-pass path; both evaluate the same chunk
 * algebra in tf32 with fp32 accumulation.  kda_verify_fwd and the fp32 /
 * KDA_FLAG_RECURRENT paths never need more than this.  Returns 0 for
 * invalid sizes.
 */
KDA_API size_t kda_chunk_fwd_workspace_size_min(int32_t N, int64_t total_T, int32_t H, int32_t d,
                                        kda_dtype dt);

/*
 * Prefill over N packed variable-length sequences (the chunked form of the
 * update rule above; the page gives only the per-token rule, the 64-token
 * chunking is this library's and reproduces the per-token result).
 *
 *   q, k, v       [total_T, H, d]  dtype dt
 *   g             [total_T, H, d]  fp32, log(alpha), finite, <= 0
 *                 ([total_T, H] with KDA_FLAG_SCALAR_DECAY)
 *   beta          [total_T, H]     fp32
 *   cu_seqlens    [N + 1] int32 DEVICE array: cu[0] = 0, non-decreasing,
 *                 cu[N] = total_T; sequence n is tokens cu[n] .. cu[n+1]-1.
 *                 Not checked on the host; an inconsistent array sets
 *                 KDA_DEVERR_CU_SEQLENS in the workspace and the offending
 *                 sequences are skipped.
 *   scale         o = scale * S^T q.
 *   flags         KDA_FLAG_*.
 *   initial_state [N, H, d, d] fp32 or NULL (= zeros).
 *   final_state   [N, H, d, d] fp32 or NULL (not written).  May alias
 *                 initial_state (in-place continuation).  A zero-length
 *                 sequence gets final = initial.
 *   o             [total_T, H, d] fp32, written for every token.
 *   workspace     device scratch of at least
 *                 kda_chunk_fwd_workspace_size_min(...) bytes (with
 *                 kda_chunk_fwd_workspace_size(...) bytes the two-pass path
 *                 runs); its first word is cleared by this call and receives
 *                 KDA_DEVERR_* bits.  Calls that share a workspace must be
 *                 stream-ordered.
 */
KDA_API int kda_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                  const float *beta, const int32_t *cu_seqlens, int32_t N, int64_t total_T,
                  int32_t H, int32_t d, kda_dtype dt, float scale, uint32_t flags,
                  const float *initial_state, float *final_state, float *o, void *workspace,
                  size_t workspace_bytes, kda_stream_t stream);

/*
 * One decode step for N sequences: each (sequence, head) state advances by
 * exactly one token, in place, and o receives that token's output
 * (o = scale * S_new^T q).  Same rule as above with T = 1.
 *
 *   q, k, v  [N, H, d] dtype dt      g [N, H, d] fp32 ([N, H] with
 *            KDA_FLAG_SCALAR_DECAY)    beta [N, H] fp32
 *   state    [N, H, d, d] fp32, read and overwritten
 *   o        [N, H, d] fp32
 */
KDA_API int kda_decode_step(const void *q, const void *k, const void *v, const float *g,
                    const float *beta, float *state, float *o, int32_t N, int32_t H,
                    int32_t d, kda_dtype dt, float scale, uint32_t flags,
                    kda_stream_t stream);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd for callers that cannot allocate
 * device memory at all (code running inside an allocator's own callbacks, an
 * embedding runtime that owns every device byte, or a service that forbids
 * allocation after start-up).  The reference pages have no counterpart: this
 * is a packaging of the same prefill.
 *
 * Same arguments and result as kda_chunk_fwd, minus the workspace: its
 * scratch is a fixed 64 KiB array inside the library (every GPU that loads
 * libkda holds it until the process exits), enough for N up to
 * KDA_NOALLOC_MAX_SEQS sequences; larger N returns KDA_ERR_WORKSPACE and
 * launches nothing.  The first call on each device looks up the array's
 * device address (with that device current), so make that first call before
 * any stream capture.  All calls share the array: it keeps the last call's
 * contents, its error word is cleared at the start of each call and cannot be
 * read back (use kda_chunk_fwd when you need it), and calls that overlap on
 * the GPU race on it -- order them on one stream.  Nothing is allocated or
 * freed.
 */
#define KDA_NOALLOC_MAX_SEQS 16320
KDA_API int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const int32_t *cu_seqlens, int32_t N,
                          int64_t total_T, int32_t H, int32_t d, kda_dtype dt, float scale,
                          uint32_t flags, const float *initial_state, float *final_state,
                          float *o, kda_stream_t stream);

/*
 * State-pool ("slot") forms for continuous batching: instead of a dense
 * [N, H, d, d] state array, the states live in a pool
 *   state_pool [num_slots, H, d, d] fp32
 * and sequence n uses the entry slots[n] (slots: [N] int32 DEVICE array,
 * distinct values in [0, num_slots); two sequences sharing a slot race).
 * The pages have no interface at all; the pool only changes where states are
 * read and written, not the arithmetic.
 *
 * kda_chunk_fwd_slots: as kda_chunk_fwd with initial_state = final_state =
 * state_pool[slots[n]] (the state is read and updated in place; clear a slot
 * before starting a new sequence in it).  A slot outside [0, num_slots) sets
 * KDA_DEVERR_SLOT in the workspace and that sequence is skipped.
 */
KDA_API int kda_chunk_fwd_slots(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const int32_t *cu_seqlens, int32_t N,
                        int64_t total_T, int32_t H, int32_t d, kda_dtype dt, float scale,
                        uint32_t flags, float *state_pool, const int32_t *slots,
                        int32_t num_slots, float *o, void *workspace, size_t workspace_bytes,
                        kda_stream_t stream);

/*
 * kda_decode_step_slots: as kda_decode_step with state = state_pool[slots[n]],
 * updated in place.  A sequence whose slot is outside [0, num_slots) is
 * skipped: no state is read or written for it, and its o rows are set to NaN
 * so that the skip shows in the output (decode has no workspace to report it
 * in).
 */
KDA_API int kda_decode_step_slots(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *state_pool, const int32_t *slots,
                          int32_t num_slots, float *o, int32_t N, int32_t H, int32_t d,
                          kda_dtype dt, float scale, uint32_t flags, kda_stream_t stream);

/*
 * kda_verify_fwd -- multi-token step for speculative decoding: each sequence
 * advances by its (few) draft tokens and the state after EVERY token is kept,
 * so the caller can roll back to the longest accepted prefix (the state after
 * token cu[n] + a - 1, or the initial state when a = 0).  Page "18B Active
 * for Just $0.045: How GLM-5.3-Flash Beat Claude with Hybrid Attention"
 * (kongchang.com), section "The Architecture Stack", names one MTP draft layer
 * for speculative decoding and the text after it describes draft, parallel
 * verify and rollback; the arithmetic is the same update rule.
 *
 * Arguments as kda_chunk_fwd (no final_state), plus
 *   state_snapshots [total_T, H, d, d] fp32: the state after each token.
 * Runs the token-by-token fp32 kernel (64 KiB written per token and head).
 */
KDA_API int kda_verify_fwd(const void *q, const void *k, const void *v, const float *g,
                   const float *beta, const int32_t *cu_seqlens, int32_t N, int64_t total_T,
                   int32_t H, int32_t d, kda_dtype dt, float scale, uint32_t flags,
                   const float *initial_state, float *state_snapshots, float *o,
                   void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * Copy the device error word of a workspace used by kda_chunk_fwd to *out
 * (synchronises `stream`).  Returns KDA_OK or KDA_ERR_*.
 */
KDA_API int kda_workspace_error(const void *workspace, uint32_t *out, kda_stream_t stream);

/*
 * Self-test of the kernels' bounded waits (no counterpart on the pages; it
 * exists so that the failure path can be exercised without a GPU fault).
 * Launches one small kernel that waits, `polls` times at most each, for a
 * global flag that nothing sets (workspace word 1, cleared by this call) and
 * for an mbarrier phase that never completes; each wait that gives up sets
 * KDA_DEVERR_TIMEOUT in workspace word 0 (cleared by this call) and the
 * kernel returns normally, so the context stays usable.  workspace: device
 * memory, 16-byte aligned, at least 256 bytes.  Returns KDA_OK once the
 * kernel is enqueued; read the outcome with kda_workspace_error().
 */
KDA_API int kda_selftest_bounded_waits(void *workspace, size_t workspace_bytes, uint32_t polls,
                                       kda_stream_t stream);

/*
 * kda_topk_indices -- the selection step of the lightning indexer (page
 * "GLM-5.3-FLASH", dimsnsums.com, section "How can a layer search the whole
 * history selectively?": the indexer of a sparse layer scores all earlier
 * tokens and passes only the best 2,048 on to full attention).  The page defines neither the
 * score nor ties, so the scores are the caller's and the ranking is stated
 * here: a higher score ranks higher; equal scores (-0 == +0) rank the lower
 * index higher, which makes the kept set unique.
 *
 *   scores       [rows, ld] fp32 DEVICE array, 4-byte aligned, ld >= n (any
 *                row stride); row r's scores are scores[r * ld + 0 .. n_r - 1].
 *                NaN is not a score: a row holding NaN gets an unspecified
 *                selection.
 *   rows         query rows, 0 .. 65535.
 *   n            tokens per row, < 2^31.
 *   k            kept per row, 1 .. KDA_TOPK_MAX_K (2,048 on the page).
 *   row_lengths  [rows] int32 DEVICE array or NULL: n_r = clamp(row_lengths[r],
 *                0, n) (e.g. a causal prefill, where query r sees fewer
 *                tokens); NULL: n_r = n.
 *   indices      [rows, k] int32 out: the kept indices best first (descending
 *                score, then ascending index); slots past n_r hold -1.
 *   values       [rows, k] fp32 out or NULL: the kept scores in the same order
 *                (-inf in the empty slots).
 *   indices / values / row_lengths: 4-byte aligned.
 *   workspace    device scratch of kda_topk_workspace_size(rows, n, k) bytes,
 *                256-byte aligned; its first word is cleared by the call.
 * Returns KDA_OK once the kernels are enqueued, KDA_ERR_INVALID_ARG /
 * _UNSUPPORTED / _MISALIGNED / _WORKSPACE for bad arguments (nothing is
 * launched then).  The scores are read twice when the cut falls in a part of
 * the score range that holds at most 16,384 of the row's tokens (the usual
 * case), and a few more times otherwise.
 */
#define KDA_TOPK_MAX_K 4096
KDA_API size_t kda_topk_workspace_size(int32_t rows, int64_t n, int32_t k);
KDA_API int kda_topk_indices(const float *scores, int64_t ld, int32_t rows, int64_t n, int32_t k,
                             const int32_t *row_lengths, int32_t *indices, float *values,
                             void *workspace, size_t workspace_bytes, kda_stream_t stream);

/* Static English description of a kda_status value. */
KDA_API const char *kda_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* KDA_H */
