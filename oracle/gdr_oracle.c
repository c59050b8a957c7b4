/*
 * gdr_oracle.c -- plain, slow, fp64 CPU oracle of the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the
 * CUDA library is checked against.  It shares no code, header, table or
 * helper with the CUDA path, and the product never links or calls it: only
 * the tests, the smoke check and the CPU-baseline leg of the benchmark do.
 *
 * What it computes (token by token, no chunking, no reordering):
 *
 *   For every batch row b and value head h, with key head kh = h / (Nv/Nk)
 *   (the repeat_interleave grouping of the transformers GatedDeltaNet layer,
 *   blog.xlworkshop.ltd "gated-delta-net", the repeat_interleave step before
 *   torch_recurrent_gated_delta_rule), state S in R^{Dk x Dv} row-major:
 *
 *     for t = 0 .. L_b - 1:
 *        x = scale * q[b,kh,t,:]              (query scaled before the math,
 *                                               lite_boost recurrent_gated_delta_rule,
 *                                               parameter scale_value)
 *        y = k[b,kh,t,:]
 *        S[i,:] *= exp(g[b,h,t]) * exp(gk[b,h,t,i])   (decay first:
 *                                               inferencelayer deltanet.rs, delta_step
 *                                               and its decay-before-readout unit test;
 *                                               gk: lite_boost recurrent op, "gk")
 *        m = y^T S                            (kv_mem, the readout)
 *        d = beta[b,h,t] * (v[b,h,t,:] - m)   (delta)
 *        S += y d^T                           (rank-1 write)
 *        out[b,h,t,:] = x^T S                 (output after the write)
 *     out[b,h,t,:] = 0 for t >= L_b           (padding written as zero:
 *                                               lite_boost chunk_gated_delta_rule,
 *                                               actual_seq_lengths)
 *
 * The same order appears in torch_recurrent_gated_delta_rule (blog page,
 * token loop) and in the docstring of deltanet.rs.  Every quantity is double.
 * Each (b, h) chain is independent; OpenMP runs chains in parallel, and each
 * chain is computed in a fixed order, so results do not depend on the thread
 * count.
 *
 * Build: gcc -O2 -fopenmp -fPIC -shared (no -ffast-math: libm exp/log1p).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_SHAPE 1
#define ORACLE_BAD_INDEX 2
#define ORACLE_NO_MEMORY 3

/* Row normalisation with eps inside the square root:
 * x / sqrt(sum x^2 + eps) (deltanet.rs, l2norm; the transformers fallback
 * calls l2norm(x, eps=1e-6) on q and k). */
static void l2norm_row(double *x, int n, double eps) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    double inv = 1.0 / sqrt(ss + eps);
    for (int i = 0; i < n; ++i) x[i] *= inv;
}

/* softplus(z) = log(1 + e^z), written in the overflow-free exact form
 * max(z, 0) + log1p(e^{-|z|}).  (deltanet.rs uses cut-offs at +-20; the
 * exact form differs from those by under 2e-9 relative.) */
static double softplus_exact(double z) {
    return (z > 0.0 ? z : 0.0) + log1p(exp(-fabs(z)));
}

/*
 * Prologue of the layer, in fp64:
 *   q_hat = l2norm(q), k_hat = l2norm(k)          (rows of length Dk)
 *   beta  = 1 / (1 + e^{-b})                       (b.sigmoid())
 *   g     = -exp(A_log[h]) * softplus(a + dt_bias[h])
 * Sources: transformers GatedDeltaNet forward (blog page, the lines computing
 * beta and g) and deltanet.rs module docstring.  Each output pointer may be
 * NULL to skip that output.  q,k: (B, Nk, S, Dk); b, a: (B, Nv, S);
 * A_log, dt_bias: (Nv).
 */
void gdr_oracle_prologue(const double *q, const double *k, const double *b,
                         const double *a, const double *A_log,
                         const double *dt_bias, double eps, int B, int Nk,
                         int Nv, int S, int Dk, double *q_hat, double *k_hat,
                         double *beta, double *g) {
    size_t nrow = (size_t)B * Nk * S;
    if (q_hat) {
        memcpy(q_hat, q, nrow * Dk * sizeof(double));
        for (size_t r = 0; r < nrow; ++r) l2norm_row(q_hat + r * Dk, Dk, eps);
    }
    if (k_hat) {
        memcpy(k_hat, k, nrow * Dk * sizeof(double));
        for (size_t r = 0; r < nrow; ++r) l2norm_row(k_hat + r * Dk, Dk, eps);
    }
    size_t nv = (size_t)B * Nv * S;
    if (beta)
        for (size_t i = 0; i < nv; ++i) beta[i] = 1.0 / (1.0 + exp(-b[i]));
    if (g) {
        for (int bb = 0; bb < B; ++bb)
            for (int h = 0; h < Nv; ++h)
                for (int t = 0; t < S; ++t) {
                    size_t i = ((size_t)bb * Nv + h) * S + t;
                    g[i] = -exp(A_log[h]) * softplus_exact(a[i] + dt_bias[h]);
                }
    }
}

/*
 * One token of the rule on one head.  S (Dk x Dv, row-major) is updated in
 * place and o (Dv) receives x^T S after the write.  gk_row may be NULL.
 * x is the already-scaled query.
 */
static void token_step(double *S, const double *x, const double *y,
                       const double *v, double beta, double g,
                       const double *gk_row, int Dk, int Dv, double *m,
                       double *o) {
    double alpha = exp(g);
    for (int i = 0; i < Dk; ++i) {
        double f = alpha * (gk_row ? exp(gk_row[i]) : 1.0);
        double *row = S + (size_t)i * Dv;
        for (int j = 0; j < Dv; ++j) row[j] *= f;
    }
    for (int j = 0; j < Dv; ++j) m[j] = 0.0;
    for (int i = 0; i < Dk; ++i) {
        const double *row = S + (size_t)i * Dv;
        for (int j = 0; j < Dv; ++j) m[j] += y[i] * row[j];
    }
    for (int j = 0; j < Dv; ++j) m[j] = beta * (v[j] - m[j]); /* m now holds delta */
    for (int i = 0; i < Dk; ++i) {
        double *row = S + (size_t)i * Dv;
        for (int j = 0; j < Dv; ++j) row[j] += y[i] * m[j];
    }
    for (int j = 0; j < Dv; ++j) o[j] = 0.0;
    for (int i = 0; i < Dk; ++i) {
        const double *row = S + (size_t)i * Dv;
        for (int j = 0; j < Dv; ++j) o[j] += x[i] * row[j];
    }
}

/*
 * Semantics of the chunked-prefill call (lite_boost chunk_gated_delta_rule):
 * BNSD inputs, GQA, variable lengths, zero padding, optional gate and
 * initial state.  The oracle reaches the result token by token; the chunked
 * method reaches the same value up to rounding.
 *
 *   q, k           (B, Nk, S, Dk)
 *   v              (B, Nv, S, Dv)
 *   beta           (B, Nv, S)
 *   g              (B, Nv, S) or NULL (no decay, alpha = 1)
 *   initial_state  (B, Nv, Dk, Dv) or NULL (zeros)
 *   lengths        (B) or NULL (all S); each must lie in [0, S]
 *   out            (B, Nv, S, Dv)
 *   final_state    (B, Nv, Dk, Dv) or NULL
 * Returns 0, or ORACLE_BAD_SHAPE for Nv % Nk != 0 / bad sizes / a length
 * outside [0, S].
 */
int gdr_oracle_chunk_fwd(const double *q, const double *k, const double *v,
                         const double *beta, const double *g,
                         const double *initial_state, const int32_t *lengths,
                         double scale, int B, int Nk, int Nv, int S, int Dk,
                         int Dv, double *out, double *final_state) {
    if (B < 0 || Nk <= 0 || Nv <= 0 || S < 0 || Dk <= 0 || Dv <= 0) return ORACLE_BAD_SHAPE;
    if (Nv % Nk != 0) return ORACLE_BAD_SHAPE;
    if (lengths)
        for (int b = 0; b < B; ++b)
            if (lengths[b] < 0 || lengths[b] > S) return ORACLE_BAD_SHAPE;
    const int group = Nv / Nk;
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * Nv; ++bh) {
        int b = bh / Nv, h = bh % Nv, kh = h / group;
        int L = lengths ? lengths[b] : S;
        size_t sd = (size_t)Dk * Dv;
        double *St = (double *)malloc(sd * sizeof(double));
        double *x = (double *)malloc((size_t)Dk * sizeof(double));
        double *m = (double *)malloc((size_t)Dv * sizeof(double));
        if (!St || !x || !m) {
            free(St); free(x); free(m);
#pragma omp atomic write
            status = ORACLE_NO_MEMORY;
            continue;
        }
        if (initial_state)
            memcpy(St, initial_state + (size_t)bh * sd, sd * sizeof(double));
        else
            memset(St, 0, sd * sizeof(double));
        for (int t = 0; t < S; ++t) {
            double *o = out + ((size_t)bh * S + t) * Dv;
            if (t >= L) {
                for (int j = 0; j < Dv; ++j) o[j] = 0.0;
                continue;
            }
            const double *qr = q + (((size_t)b * Nk + kh) * S + t) * Dk;
            const double *kr = k + (((size_t)b * Nk + kh) * S + t) * Dk;
            const double *vr = v + ((size_t)bh * S + t) * Dv;
            size_t gi = (size_t)bh * S + t;
            for (int i = 0; i < Dk; ++i) x[i] = scale * qr[i];
            token_step(St, x, kr, vr, beta[gi], g ? g[gi] : 0.0, NULL, Dk, Dv, m, o);
        }
        if (final_state) memcpy(final_state + (size_t)bh * sd, St, sd * sizeof(double));
        free(St); free(x); free(m);
    }
    return status;
}

/*
 * Semantics of the decode call (lite_boost recurrent_gated_delta_rule):
 * a pool of state slots, one slot index per flattened token, per-key gate gk,
 * and num_accepted_tokens.
 *
 *   q, k        (B, Nk, S, Dk);  v (B, Nv, S, Dv);  beta, g (B, Nv, S)
 *   gk          (B, Nv, S, Dk) or NULL;  g may be NULL (no decay)
 *   pool        (slots, Nv, Dk, Dv), read and updated in place
 *   indices     (B*S): slot of token (b, t) is indices[b*S + t]
 *   lengths     (B): tokens of sequence b that are processed, in [0, S]
 *   accepted    (B) or NULL (= lengths)
 *   out         (B, Nv, S, Dv); rows t >= L_b are zero
 *
 * Reading of num_accepted_tokens (the page defines it only as the number of
 * accepted tokens, equal to the lengths in plain inference), per_token = 0:
 * the chain starts from pool[indices[b*S]]; all L_b tokens are processed and
 * output; the state after token t is written to pool[indices[b*S + t]] only
 * when t < min(A_b, L_b).  per_token = 1 (the speculative-decoding reading):
 * A_b counts the tokens of the previous step that were accepted, whose states
 * went to their own slots, so the chain starts from pool[indices[b*S + A_b - 1]]
 * and the state after every token t < L_b is written to pool[indices[b*S + t]];
 * A_b must lie in [1, S] (ORACLE_BAD_SHAPE otherwise; NULL accepted means 1).
 * A sequence with L_b = 0 leaves the pool untouched.
 * Returns ORACLE_BAD_INDEX for a referenced slot outside [0, slots), and
 * ORACLE_BAD_SHAPE for bad sizes or lengths outside [0, S].  Two sequences
 * must not share a slot (their chains would race; the result is undefined).
 */
int gdr_oracle_recurrent_step(const double *q, const double *k, const double *v,
                              const double *beta, const double *g,
                              const double *gk, double *pool, int slots,
                              const int32_t *indices, const int32_t *lengths,
                              const int32_t *accepted, int per_token, double scale,
                              int B, int Nk, int Nv, int S, int Dk, int Dv,
                              double *out) {
    if (B < 0 || Nk <= 0 || Nv <= 0 || S < 0 || Dk <= 0 || Dv <= 0 || slots < 0)
        return ORACLE_BAD_SHAPE;
    if (Nv % Nk != 0) return ORACLE_BAD_SHAPE;
    for (int b = 0; b < B; ++b) {
        if (lengths[b] < 0 || lengths[b] > S) return ORACLE_BAD_SHAPE;
        if (per_token && lengths[b] > 0) {
            int A = accepted ? accepted[b] : 1;
            if (A < 1 || A > S) return ORACLE_BAD_SHAPE;
            int s = indices[(size_t)b * S + A - 1];
            if (s < 0 || s >= slots) return ORACLE_BAD_INDEX;
        }
        for (int t = 0; t < lengths[b]; ++t) {
            int s = indices[(size_t)b * S + t];
            if (s < 0 || s >= slots) return ORACLE_BAD_INDEX;
        }
    }
    const int group = Nv / Nk;
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * Nv; ++bh) {
        int b = bh / Nv, h = bh % Nv, kh = h / group;
        int L = lengths[b];
        int A = accepted ? accepted[b] : (per_token ? 1 : L);
        /* commits: tokens t < ncommit; the chain starts from the slot of token `first` */
        int ncommit = per_token ? L : (A < L ? A : L);
        int first = per_token ? A - 1 : 0;
        size_t sd = (size_t)Dk * Dv;
        for (int t = L; t < S; ++t) {
            double *o = out + ((size_t)bh * S + t) * Dv;
            for (int j = 0; j < Dv; ++j) o[j] = 0.0;
        }
        if (L == 0) continue;
        double *St = (double *)malloc(sd * sizeof(double));
        double *x = (double *)malloc((size_t)Dk * sizeof(double));
        double *m = (double *)malloc((size_t)Dv * sizeof(double));
        if (!St || !x || !m) {
            free(St); free(x); free(m);
#pragma omp atomic write
            status = ORACLE_NO_MEMORY;
            continue;
        }
        int s0 = indices[(size_t)b * S + first];
        memcpy(St, pool + ((size_t)s0 * Nv + h) * sd, sd * sizeof(double));
        for (int t = 0; t < L; ++t) {
            const double *qr = q + (((size_t)b * Nk + kh) * S + t) * Dk;
            const double *kr = k + (((size_t)b * Nk + kh) * S + t) * Dk;
            const double *vr = v + ((size_t)bh * S + t) * Dv;
            size_t gi = (size_t)bh * S + t;
            const double *gkr = gk ? gk + gi * Dk : NULL;
            double *o = out + gi * Dv;
            for (int i = 0; i < Dk; ++i) x[i] = scale * qr[i];
            token_step(St, x, kr, vr, beta[gi], g ? g[gi] : 0.0, gkr, Dk, Dv, m, o);
            if (t < ncommit) {
                int st = indices[(size_t)b * S + t];
                memcpy(pool + ((size_t)st * Nv + h) * sd, St, sd * sizeof(double));
            }
        }
        free(St); free(x); free(m);
    }
    return status;
}

/* Sets the number of OpenMP threads of later calls (for a single-thread timing); n < 1 is ignored.  The
 * results do not depend on it: every chain is computed in the same fixed order. */
void gdr_oracle_set_threads(int n) {
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Number of OpenMP threads the oracle will use (reported with timings). */
int gdr_oracle_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
