/*
 * Gated Delta Rule-2 oracle: plain, sequential, fp64, token by token.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may include, link
 * or call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline use it. It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes (per sequence n and head h, state S in R^{d_k x d_v}):
 *
 *   S_t = (I - k_t (b_t . k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T
 *   o_t = S_t^T q_t
 *
 * with alpha_t = exp(log_alpha_t) a per-key-channel decay. Sources:
 *   - "Gated DeltaNet-2: Decoupling Erase and Write Gates in Linear Attention
 *     for Better Memory Editing" (zhichai.net forum summary), section
 *     "Gated Delta Rule-2": the update rule, erase gate b_t in [0,1]^{d_k},
 *     write gate w_t in [0,1]^{d_v}, z_t = w_t . v_t, e_t = b_t . k_t.
 *   - The same article in Chinese (zhichai.net), section
 *     "Gated Delta Rule-2: 擦除和写入，各走各的路": the same update rule.
 *   - "엔비디아, 기억 수정 최적화 선형 어텐션 모델 공개" (ainews.random.gg),
 *     section "Gated Delta Rule-2: two gates instead of one": D_t =
 *     Diag(alpha_t) is channel-wise over key channels, the decay is applied
 *     before the active edit, and the layer "stores a matrix state S_t and
 *     reads it with the query" (readout from the post-update state).
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - layouts: token tensors are token-major [B, T, H, d]; the state is
 *     [N, H, d_k, d_v] with d_v contiguous;
 *   - no scale on q, no activation or normalisation inside the operator;
 *   - the readout uses the post-update state;
 *   - with cu_seqlens, token tensors are [1, T_total, H, d] and sequence n
 *     covers tokens cu_seqlens[n] .. cu_seqlens[n+1]-1.
 *
 * The step is written exactly as the rule reads, one operation at a time:
 * decay the rows, read the old content along the gated erase direction e_t,
 * subtract it along k_t and add the gated write, then read out with q_t.
 * Parallelism, when requested, is only across independent (sequence, head)
 * units; each unit's arithmetic is the same sequential loop.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One token of the recurrence on a single (sequence, head) state.
 * S: d_k x d_v row-major (updated in place); q, k, la, b: length d_k;
 * v, w: length d_v; o: length d_v (output); scratch: 2*d_v doubles. */
static void gdr2_token(double *S, const double *q, const double *k,
                       const double *la, const double *b, const double *v,
                       const double *w, double *o, int64_t dk, int64_t dv,
                       double *scratch)
{
    double *read = scratch;      /* e_t^T (D_t S_{t-1}), length d_v */
    double *resid = scratch + dv; /* z_t - read, length d_v        */

    /* D_t S_{t-1}: decay each key row c by alpha_{t,c} (before the edit). */
    for (int64_t c = 0; c < dk; ++c) {
        double a = exp(la[c]);
        double *row = S + c * dv;
        for (int64_t j = 0; j < dv; ++j) row[j] *= a;
    }
    /* read_j = sum_c e_c S[c][j] with e = b . k (gated erase direction). */
    for (int64_t j = 0; j < dv; ++j) read[j] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
        double e = b[c] * k[c];
        const double *row = S + c * dv;
        for (int64_t j = 0; j < dv; ++j) read[j] += e * row[j];
    }
    /* S <- S - k read^T + k z^T  with z = w . v (gated write target). */
    for (int64_t j = 0; j < dv; ++j) resid[j] = w[j] * v[j] - read[j];
    for (int64_t c = 0; c < dk; ++c) {
        double *row = S + c * dv;
        for (int64_t j = 0; j < dv; ++j) row[j] += k[c] * resid[j];
    }
    /* o_t = S_t^T q_t (post-update readout). */
    for (int64_t j = 0; j < dv; ++j) o[j] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
        const double *row = S + c * dv;
        for (int64_t j = 0; j < dv; ++j) o[j] += q[c] * row[j];
    }
}

/* Whole-sequence forward.
 * Token tensors (q, k, log_alpha, b: [B,T,H,d_k]; v, w, o: [B,T,H,d_v]) are
 * token-major. With cu_seqlens (length num_seqs+1, non-decreasing, first 0),
 * B must be 1 and sequence n spans tokens cu_seqlens[n]..cu_seqlens[n+1]-1;
 * otherwise num_seqs = B and every sequence has length T.
 * init_state / final_state: [num_seqs, H, d_k, d_v]; init_state may be NULL
 * (zeros), final_state may be NULL (not written).
 * num_threads <= 0 uses the OpenMP default. Returns 0 on success, -1 on bad
 * arguments, -2 on allocation failure. */
int gdr2_oracle_forward(const double *q, const double *k, const double *v,
                        const double *log_alpha, const double *b,
                        const double *w, const double *init_state,
                        const int64_t *cu_seqlens, int64_t B, int64_t T,
                        int64_t H, int64_t dk, int64_t dv, int64_t num_seqs,
                        double *o, double *final_state, int num_threads)
{
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    if (cu_seqlens) {
        if (B != 1 || num_seqs < 0 || cu_seqlens[0] != 0 ||
            cu_seqlens[num_seqs] != T)
            return -1;
        for (int64_t n = 0; n < num_seqs; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    } else if (num_seqs != B) {
        return -1;
    }
    const int64_t units = num_seqs * H;
    int failed = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
#endif
    for (int64_t u = 0; u < units; ++u) {
        const int64_t n = u / H, h = u % H;
        int64_t t0, t1;
        if (cu_seqlens) {
            t0 = cu_seqlens[n];
            t1 = cu_seqlens[n + 1];
        } else {
            t0 = n * T;
            t1 = n * T + T;
        }
        double *S = (double *)malloc(sizeof(double) * (size_t)(dk * dv));
        double *scratch = (double *)malloc(sizeof(double) * (size_t)(2 * dv));
        if (!S || !scratch) {
            free(S);
            free(scratch);
            failed = 1;
            continue;
        }
        if (init_state)
            memcpy(S, init_state + u * dk * dv, sizeof(double) * (size_t)(dk * dv));
        else
            memset(S, 0, sizeof(double) * (size_t)(dk * dv));
        for (int64_t t = t0; t < t1; ++t) {
            const int64_t rk = (t * H + h) * dk, rv = (t * H + h) * dv;
            gdr2_token(S, q + rk, k + rk, log_alpha + rk, b + rk, v + rv, w + rv,
                       o + rv, dk, dv, scratch);
        }
        if (final_state)
            memcpy(final_state + u * dk * dv, S, sizeof(double) * (size_t)(dk * dv));
        free(S);
        free(scratch);
    }
    return failed ? -2 : 0;
}

/* One decode step for N independent sequences: token tensors [N,H,d],
 * state [N,H,d_k,d_v] updated in place, o [N,H,d_v]. */
int gdr2_oracle_step(const double *q, const double *k, const double *v,
                     const double *log_alpha, const double *b, const double *w,
                     double *state, int64_t N, int64_t H, int64_t dk,
                     int64_t dv, double *o, int num_threads)
{
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    const int64_t units = N * H;
    int failed = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(static) reduction(| : failed)
#endif
    for (int64_t u = 0; u < units; ++u) {
        double *scratch = (double *)malloc(sizeof(double) * (size_t)(2 * dv));
        if (!scratch) {
            failed = 1;
            continue;
        }
        gdr2_token(state + u * dk * dv, q + u * dk, k + u * dk, log_alpha + u * dk,
                   b + u * dk, v + u * dv, w + u * dv, o + u * dv, dk, dv, scratch);
        free(scratch);
    }
    return failed ? -2 : 0;
}

/* ---------------------------------------------------------------------------
 * QED: a second erase direction derived from the query ("The Query Knows
 * What to Forget: A Second Erase Direction for Linear Attention",
 * thelatestinai.com listing: abstract and Table 1). The page names the parts
 * of the correction (a direction from the query, projected orthogonal to the
 * key, gated by b_t, with a per-head strength) but does not print its
 * equation (6); this is the plain reading recorded in the design notes,
 * PARITY UNPINNED against the paper (pinned only by the reading's own
 * invariants and reductions):
 *
 *   src_t = q_t, or a fixed per-head direction r_h (the control arm)
 *   p_t   = src_t - (k_t.src_t / k_t.k_t) k_t      (projection P^perp_{k_t};
 *                                                   p_t = src_t if unprojected
 *                                                   or k_t = 0)
 *   u_t   = p_t / |p_t|   (0 when |p_t|^2 <= 1e-12 |src_t|^2)
 *   f_t   = b_t . u_t     (u_t if ungated)
 *   S_t   = (I - k_t (b_t . k_t)^T - lambda_h u_t f_t^T) Diag(alpha_t) S_{t-1}
 *           + k_t (w_t . v_t)^T,           o_t = S_t^T q_t.
 *
 * flags: bit 0 gate the correction by b_t, bit 1 project orthogonal to k_t.
 * ------------------------------------------------------------------------ */
#define QED_GATE 1
#define QED_PROJECT 2

/* One QED token on one (sequence, head) state; scratch: 3*d_v + d_k doubles. */
static void qed_token(double *S, const double *q, const double *k, const double *la,
                      const double *b, const double *v, const double *w,
                      const double *dir, double lambda, int flags, double *o,
                      int64_t dk, int64_t dv, double *scratch)
{
    double *read_k = scratch;           /* (b.k)^T D S, length d_v */
    double *read_u = scratch + dv;      /* f^T D S, length d_v     */
    double *resid = scratch + 2 * dv;   /* z - read_k, length d_v  */
    double *u = scratch + 3 * dv;       /* erase direction, d_k    */

    /* D_t S_{t-1} */
    for (int64_t c = 0; c < dk; ++c) {
        double a = exp(la[c]);
        double *row = S + c * dv;
        for (int64_t j = 0; j < dv; ++j) row[j] *= a;
    }
    /* u_t: the source direction, projected orthogonal to k_t, normalised */
    const double *src = dir ? dir : q;
    double kk = 0.0, ks = 0.0, ss = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
        kk += k[c] * k[c];
        ks += k[c] * src[c];
        ss += src[c] * src[c];
    }
    double coef = ((flags & QED_PROJECT) && kk > 0.0) ? ks / kk : 0.0;
    double pp = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
        u[c] = src[c] - coef * k[c];
        pp += u[c] * u[c];
    }
    double inv = (pp > 1e-12 * ss && pp > 0.0) ? 1.0 / sqrt(pp) : 0.0;
    for (int64_t c = 0; c < dk; ++c) u[c] *= inv;
    /* both reads of the decayed state, before either edit */
    for (int64_t j = 0; j < dv; ++j) read_k[j] = read_u[j] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
        double e = b[c] * k[c];
        double f = (flags & QED_GATE) ? b[c] * u[c] : u[c];
        const double *row = S + c * dv;
        for (int64_t j = 0; j < dv; ++j) {
            read_k[j] += e * row[j];
            read_u[j] += f * row[j];
        }
    }
    /* S <- S - k read_k^T - lambda u read_u^T + k z^T */
    for (int64_t j = 0; j < dv; ++j) resid[j] = w[j] * v[j] - read_k[j];
    for (int64_t c = 0; c < dk; ++c) {
        double *row = S + c * dv;
        double lu = lambda * u[c];
        for (int64_t j = 0; j < dv; ++j) row[j] += k[c] * resid[j] - lu * read_u[j];
    }
    /* o_t = S_t^T q_t */
    for (int64_t j = 0; j < dv; ++j) o[j] = 0.0;
    for (int64_t c = 0; c < dk; ++c) {
        const double *row = S + c * dv;
        for (int64_t j = 0; j < dv; ++j) o[j] += q[c] * row[j];
    }
}

/* Whole-sequence QED forward; arguments as gdr2_oracle_forward, plus
 * lambda [H] (per-head strength), dir [H, d_k] (fixed directions, or NULL for
 * the query) and flags. */
int gdr2_oracle_qed_forward(const double *q, const double *k, const double *v,
                            const double *log_alpha, const double *b,
                            const double *w, const double *lambda, const double *dir,
                            int flags, const double *init_state,
                            const int64_t *cu_seqlens, int64_t B, int64_t T,
                            int64_t H, int64_t dk, int64_t dv, int64_t num_seqs,
                            double *o, double *final_state, int num_threads)
{
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0 || !lambda) return -1;
    if (cu_seqlens) {
        if (B != 1 || num_seqs < 0 || cu_seqlens[0] != 0 ||
            cu_seqlens[num_seqs] != T)
            return -1;
        for (int64_t n = 0; n < num_seqs; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    } else if (num_seqs != B) {
        return -1;
    }
    const int64_t units = num_seqs * H;
    int failed = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
#endif
    for (int64_t u = 0; u < units; ++u) {
        const int64_t n = u / H, h = u % H;
        int64_t t0 = cu_seqlens ? cu_seqlens[n] : n * T;
        int64_t t1 = cu_seqlens ? cu_seqlens[n + 1] : n * T + T;
        double *S = (double *)malloc(sizeof(double) * (size_t)(dk * dv));
        double *scratch = (double *)malloc(sizeof(double) * (size_t)(3 * dv + dk));
        if (!S || !scratch) {
            free(S);
            free(scratch);
            failed = 1;
            continue;
        }
        if (init_state)
            memcpy(S, init_state + u * dk * dv, sizeof(double) * (size_t)(dk * dv));
        else
            memset(S, 0, sizeof(double) * (size_t)(dk * dv));
        for (int64_t t = t0; t < t1; ++t) {
            const int64_t rk = (t * H + h) * dk, rv = (t * H + h) * dv;
            qed_token(S, q + rk, k + rk, log_alpha + rk, b + rk, v + rv, w + rv,
                      dir ? dir + h * dk : NULL, lambda[h], flags, o + rv, dk, dv, scratch);
        }
        if (final_state)
            memcpy(final_state + u * dk * dv, S, sizeof(double) * (size_t)(dk * dv));
        free(S);
        free(scratch);
    }
    return failed ? -2 : 0;
}

/* Number of threads an OpenMP parallel region would use (1 without OpenMP). */
int gdr2_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
