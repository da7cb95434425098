/*
 * kda_oracle.c -- plain fp64 CPU reference of the Kimi Delta Attention (KDA)
 * recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may link,
 * load or call this file: only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or table with the CUDA
 * implementation.
 *
 * What it computes (page "GLM-5.3-FLASH" at dimsnsums.com/models/glm-5-3-flash/
 * attention, section "How can a layer remember without rereading?", the
 * displayed update rule):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *
 * per head, with S a d_k x d_v = 128 x 128 matrix whose ROWS are key channels
 * (alpha_t multiplies S from the left, so each of the 128 key channels decays
 * at its own rate; the same section states the per-channel decay in prose).
 * The readout o_t = scale * S_t^T q_t (the page's "one summary read") uses the
 * state after token t's update.  The page writes beta, k, v without a token
 * index; they are read as per-token quantities like alpha_t.
 *
 * Expanding the product gives the form evaluated here, token by token:
 *     S'  = Diag(alpha_t) S_{t-1}          (decay each key row)
 *     u   = S'^T k_t                       (what the state recalls for k_t)
 *     S_t = S' + beta_t k_t (v_t - u)^T    (erase the old note, write the new one)
 *     o_t = scale * S_t^T q_t
 * which is (I - beta k k^T) S' + beta k v^T exactly (S' - beta k (k^T S')
 * + beta k v^T), so no step is reordered.
 *
 * Inputs are given as g = log(alpha) (alpha = exp(g)).  When `l2norm` is set,
 * q_t and k_t are first replaced by x / sqrt(sum(x^2) + eps) over the d
 * channels of the head.
 *
 * Layouts (row-major, fp64): q, k, v, g, o: [total_T, H, d]; beta: [total_T, H];
 * states: [N, H, d, d] with element (n, h, i, j) = row i (key channel),
 * column j (value channel); cu_seqlens: [N + 1] with sequence n occupying
 * tokens cu_seqlens[n] .. cu_seqlens[n+1]-1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static void normalise(double *dst, const double *src, int64_t d, int l2norm, double eps)
{
    if (!l2norm) {
        memcpy(dst, src, (size_t)d * sizeof(double));
        return;
    }
    double ss = 0.0;
    for (int64_t i = 0; i < d; ++i) ss += src[i] * src[i];
    double r = 1.0 / sqrt(ss + eps);
    for (int64_t i = 0; i < d; ++i) dst[i] = src[i] * r;
}

/* One token of the recurrence on state S (d x d, row = key channel). */
static void kda_token(double *S, int64_t d, const double *q_raw, const double *k_raw,
                      const double *v, const double *g, double beta, double scale,
                      int l2norm, double eps, double *o, double *work)
{
    double *q = work, *k = work + d, *u = work + 2 * d;
    normalise(q, q_raw, d, l2norm, eps);
    normalise(k, k_raw, d, l2norm, eps);

    /* S' = Diag(alpha) S : row i scaled by alpha_i = exp(g_i) */
    for (int64_t i = 0; i < d; ++i) {
        double a = exp(g[i]);
        double *row = S + i * d;
        for (int64_t j = 0; j < d; ++j) row[j] *= a;
    }
    /* u = S'^T k */
    for (int64_t j = 0; j < d; ++j) u[j] = 0.0;
    for (int64_t i = 0; i < d; ++i) {
        const double *row = S + i * d;
        double ki = k[i];
        for (int64_t j = 0; j < d; ++j) u[j] += row[j] * ki;
    }
    /* S = S' + beta k (v - u)^T */
    for (int64_t i = 0; i < d; ++i) {
        double *row = S + i * d;
        double bk = beta * k[i];
        for (int64_t j = 0; j < d; ++j) row[j] += bk * (v[j] - u[j]);
    }
    /* o = scale * S^T q */
    for (int64_t j = 0; j < d; ++j) o[j] = 0.0;
    for (int64_t i = 0; i < d; ++i) {
        const double *row = S + i * d;
        double qi = q[i];
        for (int64_t j = 0; j < d; ++j) o[j] += row[j] * qi;
    }
    for (int64_t j = 0; j < d; ++j) o[j] *= scale;
}

/*
 * Prefill over packed sequences.  Returns 0, or -1 on inconsistent sizes.
 * initial_state may be NULL (zeros); final_state may be NULL (not written).
 * o must not alias the inputs.  nthreads <= 0 means the OpenMP default.
 */
int kda_oracle_forward(int64_t N, int64_t H, int64_t d, const int64_t *cu_seqlens,
                       const double *q, const double *k, const double *v, const double *g,
                       const double *beta, const double *initial_state, double *final_state,
                       double *o, double scale, int l2norm, double eps, int nthreads)
{
    if (N < 0 || H <= 0 || d <= 0 || cu_seqlens == NULL) return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int64_t n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    const int64_t pairs = N * H;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int status = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < pairs; ++p) {
        const int64_t n = p / H, h = p % H;
        double *S = (double *)malloc((size_t)(d * d + 3 * d) * sizeof(double));
        if (!S) {
#pragma omp atomic write
            status = -2;
            continue;
        }
        double *work = S + d * d;
        if (initial_state)
            memcpy(S, initial_state + (n * H + h) * d * d, (size_t)(d * d) * sizeof(double));
        else
            memset(S, 0, (size_t)(d * d) * sizeof(double));
        for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
            const int64_t base = (t * H + h) * d;
            kda_token(S, d, q + base, k + base, v + base, g + base, beta[t * H + h], scale,
                      l2norm, eps, o + base, work);
        }
        if (final_state)
            memcpy(final_state + (n * H + h) * d * d, S, (size_t)(d * d) * sizeof(double));
        free(S);
    }
    return status;
}

/*
 * One decode step: every (sequence, head) state advances by exactly one token,
 * in place.  q, k, v, g, o: [N, H, d]; beta: [N, H]; state: [N, H, d, d].
 */
int kda_oracle_decode(int64_t N, int64_t H, int64_t d, const double *q, const double *k,
                      const double *v, const double *g, const double *beta, double *state,
                      double *o, double scale, int l2norm, double eps, int nthreads)
{
    if (N < 0 || H <= 0 || d <= 0) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int status = 0;
    const int64_t pairs = N * H;
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < pairs; ++p) {
        double *work = (double *)malloc((size_t)(3 * d) * sizeof(double));
        if (!work) {
#pragma omp atomic write
            status = -2;
            continue;
        }
        kda_token(state + p * d * d, d, q + p * d, k + p * d, v + p * d, g + p * d, beta[p],
                  scale, l2norm, eps, o + p * d, work);
        free(work);
    }
    return status;
}

/* Number of threads OpenMP would use for the next parallel region. */
int kda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
