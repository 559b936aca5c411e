/*
 * KDA recurrence oracle: plain, slow, token-by-token fp64 CPU implementation.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call this code:
 * only the tests, the package smoke check and the benchmark's CPU-baseline leg
 * load it. It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (per sequence n and head h, state S of shape d_k x d_v,
 * row c = key channel, column j = value channel), for each token t in order:
 *
 *   1. forget:  S[c][:] *= alpha[t][c],  alpha = exp(log_alpha)     (one gate per key channel)
 *   2. recall:  pred[j]  = sum_c S[c][j] * k[t][c]                  (S^T k)
 *   3. compare: err[j]   = v[t][j] - pred[j]
 *   4. correct: S[c][j] += beta[t] * k[t][c] * err[j]               (write only the error)
 *   5. read:    out[t][j] = sum_c S[c][j] * q[t][c]                 (after the write)
 *
 * Sources:
 *  - "Kimi K3 -- the architecture and infrastructure, explained" (shivam2003.com),
 *    section "How the delta rule actually works": the state predicts v from k and
 *    the update writes only the correction, S <- S - beta (S k - v) k^T. That page
 *    stores S as d_v x d_k; here S is its transpose (d_k x d_v), the same map.
 *  - same page, section "Kimi Delta Attention: the load-bearing choice", and the
 *    marketersindex.com Kimi K3 article, section "Architectural Innovations: Kimi
 *    Delta Attention (KDA)": forgetting is per channel (rows of the state decay
 *    at different speeds) -- step 1.
 *  - aitrending.vip "Inside Kimi K3", section "Technical Details": beta is the
 *    writing strength and alpha the forgetting factor, 128 forgetting dials per
 *    head -- alpha has one entry per key channel, beta one per token and head.
 *  - Readings where the pages are silent: decay is applied before the delta
 *    correction (recall sees the decayed state) and the output is read after the
 *    write; no 1/sqrt(d_k) scaling is applied inside the recurrence.
 *
 * Precision: every value is fp64; inputs arrive as fp64 copies of the exact
 * bf16/fp32 values the GPU consumed. exp() is the C library's double exp.
 *
 * Layouts (row-major, d contiguous): q, k, log_alpha [T_total][H][d_k];
 * v, out [T_total][H][d_v]; beta [T_total][H]; states [N][H][d_k][d_v];
 * cu_seqlens [N+1] token offsets of the packed sequences.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Runs the recurrence for every (sequence, head). initial_state may be NULL
 * (zero start); final_state may be NULL (not wanted). Returns 0 on success,
 * -1 on a bad argument, -2 on allocation failure. */
int kda_oracle_forward(const double *q, const double *k, const double *v,
                       const double *log_alpha, const double *beta,
                       const double *initial_state, const int64_t *cu_seqlens,
                       int32_t num_seqs, int32_t H, int32_t dk, int32_t dv,
                       double *out, double *final_state, int32_t num_threads)
{
    if (num_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens)
        return -1;
    for (int32_t n = 0; n < num_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n])
            return -1;
    const int64_t pairs = (int64_t)num_seqs * H;
    int failed = 0;
#ifdef _OPENMP
    if (num_threads > 0)
        omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
#endif
    for (int64_t p = 0; p < pairs; ++p) {
        const int64_t n = p / H, h = p % H;
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * (size_t)dv);
        double *pred = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!S || !pred) {
            free(S);
            free(pred);
            failed |= 1;
            continue;
        }
        const size_t sdim = (size_t)dk * (size_t)dv;
        if (initial_state)
            memcpy(S, initial_state + (size_t)p * sdim, sizeof(double) * sdim);
        else
            memset(S, 0, sizeof(double) * sdim);

        for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
            const double *kt = k + ((size_t)t * H + h) * dk;
            const double *qt = q + ((size_t)t * H + h) * dk;
            const double *vt = v + ((size_t)t * H + h) * dv;
            const double *lat = log_alpha + ((size_t)t * H + h) * dk;
            const double bt = beta[(size_t)t * H + h];
            /* 1. forget, channel by channel */
            for (int32_t c = 0; c < dk; ++c) {
                const double a = exp(lat[c]);
                for (int32_t j = 0; j < dv; ++j)
                    S[(size_t)c * dv + j] *= a;
            }
            /* 2. recall: pred = S^T k */
            for (int32_t j = 0; j < dv; ++j)
                pred[j] = 0.0;
            for (int32_t c = 0; c < dk; ++c)
                for (int32_t j = 0; j < dv; ++j)
                    pred[j] += S[(size_t)c * dv + j] * kt[c];
            /* 3. compare, 4. correct: S += beta k (v - pred)^T */
            for (int32_t c = 0; c < dk; ++c) {
                const double w = bt * kt[c];
                for (int32_t j = 0; j < dv; ++j)
                    S[(size_t)c * dv + j] += w * (vt[j] - pred[j]);
            }
            /* 5. read: out = S^T q */
            double *ot = out + ((size_t)t * H + h) * dv;
            for (int32_t j = 0; j < dv; ++j)
                ot[j] = 0.0;
            for (int32_t c = 0; c < dk; ++c)
                for (int32_t j = 0; j < dv; ++j)
                    ot[j] += S[(size_t)c * dv + j] * qt[c];
        }
        if (final_state)
            memcpy(final_state + (size_t)p * sdim, S, sizeof(double) * sdim);
        free(S);
        free(pred);
    }
    return failed ? -2 : 0;
}

/*
 * Influence bound for a state window (used to check the final state of a very
 * long sequence without running the whole oracle).
 *
 * With beta in [0,1] and unit keys, the per-token map S -> (I - beta k k^T) Diag(alpha) S
 * has spectral norm at most max_c alpha[c] <= 1, because (I - beta k k^T) is a
 * symmetric matrix with eigenvalues 1 - beta and 1. Hence two runs that differ
 * only in the state at the start of a window of tokens differ at its end by at
 * most prod_t max_c alpha[t][c] times the (spectral) norm of the starting
 * difference, and ||S_t||_2 <= max_c alpha[t][c] ||S_{t-1}||_2 + beta_t ||k_t|| ||v_t||.
 *
 * For one (sequence, head), over tokens [t0, t1) of the packed arrays, this
 * returns in *log_decay the sum over the window of log(max_c alpha[t][c]), and
 * in *norm_bound the running bound b on ||S||_2 at t0 obtained by iterating
 * b <- max_c alpha * b + beta ||k|| ||v|| from b = s0_norm over tokens [t_start, t0).
 * The influence of the true state at t0 on the state at t1 is then at most
 * exp(*log_decay) * (*norm_bound) in spectral norm (and so in max-abs).
 */
int kda_oracle_window_bound(const double *k, const double *v, const double *log_alpha,
                            const double *beta, int32_t H, int32_t dk, int32_t dv,
                            int32_t h, int64_t t_start, int64_t t0, int64_t t1,
                            double s0_norm, double *log_decay, double *norm_bound)
{
    if (h < 0 || h >= H || t_start > t0 || t0 > t1 || !log_decay || !norm_bound)
        return -1;
    double b = s0_norm;
    for (int64_t t = t_start; t < t0; ++t) {
        const double *lat = log_alpha + ((size_t)t * H + h) * dk;
        const double *kt = k + ((size_t)t * H + h) * dk;
        const double *vt = v + ((size_t)t * H + h) * dv;
        double mx = -INFINITY, kk = 0.0, vv = 0.0;
        for (int32_t c = 0; c < dk; ++c) {
            if (lat[c] > mx)
                mx = lat[c];
            kk += kt[c] * kt[c];
        }
        for (int32_t j = 0; j < dv; ++j)
            vv += vt[j] * vt[j];
        b = exp(mx) * b + beta[(size_t)t * H + h] * sqrt(kk) * sqrt(vv);
    }
    double ld = 0.0;
    for (int64_t t = t0; t < t1; ++t) {
        const double *lat = log_alpha + ((size_t)t * H + h) * dk;
        double mx = -INFINITY;
        for (int32_t c = 0; c < dk; ++c)
            if (lat[c] > mx)
                mx = lat[c];
        ld += mx;
    }
    *log_decay = ld;
    *norm_bound = b;
    return 0;
}

int kda_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
