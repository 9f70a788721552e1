/*
 * gptattn_oracle.c -- plain fp64 CPU oracle for batched multi-head causal
 * scaled dot-product self-attention (forward and backward).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no source, header, table or helper
 * with the CUDA kernels.
 *
 * What it computes is the plain definition, written out with no blocking,
 * fusion or reordering, following these passages:
 *
 *  - "Let's build GPT: from scratch, in code, spelled out" (lecture page),
 *    chapter "version 4: self-attention": every token emits a query, a key and
 *    a value; the affinity of token t for token s is the dot product q_t . k_s.
 *  - same page, chapter "version 3: adding softmax": affinities of one row
 *    become aggregation weights through a softmax over the row.
 *  - same page, chapters "the trick in self-attention: matrix multiply as
 *    weighted aggregation" / "version 2": the output row is the weighted sum
 *    of value rows.
 *  - same page, note 4 (decoder blocks) and the correction to 00:57:00:
 *    tokens from the future cannot communicate, so s > t is masked out;
 *    s == t stays visible (a token always sees itself).
 *  - same page, note 6 and the correction to 01:20:05: scores are divided by
 *    sqrt(head_size), not sqrt(C).
 *  - same page, exercise EX1 and chapter "batched multi-headed
 *    self-attention": all heads at once, heads treated as one more batch
 *    dimension; head h owns columns [h*hs, (h+1)*hs) of each of q, k, v.
 *  - same page, note 3: no communication across the batch dimension.
 *  - minGPT README page ("卡帕西(氏)MinGPT"), reference notes on GPT-3: the
 *    layers alternate dense attention with locally banded sparse attention
 *    (no band width is given).  Read here as a local window of `window`
 *    positions: token t sees s with t - window < s <= t (itself and the
 *    window-1 before it); window >= T is the dense causal case above, with the
 *    same arithmetic.
 *
 * Input packing (the projection output of a GPT-2 style block): qkv[B][T][3C]
 * row-major, q = columns [0,C), k = [C,2C), v = [2C,3C).  Output y[B][T][C]
 * (heads concatenated back along C), lse[B][n_head][T] (natural log of the
 * softmax normaliser of each row, i.e. logsumexp of the masked scaled scores).
 *
 * Backward: given dy = dL/dy, the chain rule through the three steps above
 * (weighted sum, softmax, scaled dot product) gives
 *     dV = P^T dY,   dP = dY V^T,   dS = P o (dP - rowsum(P o dP)),
 *     dQ = dS K / sqrt(hs),   dK = dS^T Q / sqrt(hs),
 * packed into dqkv[B][T][3C] with the same layout as qkv.
 *
 * All arithmetic is IEEE double.  Work is split across (batch, head) pairs
 * with OpenMP; each pair is computed by one thread in plain loops.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

static int check_shape(int B, int T, int C, int n_head) {
    if (B < 0 || T < 0 || C <= 0 || n_head <= 0) return ORACLE_EINVAL;
    if (C % n_head != 0) return ORACLE_EINVAL;
    return ORACLE_OK;
}

/* Element d of the q (part 0), k (part 1) or v (part 2) row of head h at
 * position t of batch b. */
static inline double qkv_at(const double *qkv, int T, int C, int hs, int b, int t,
                            int part, int h, int d) {
    size_t row = (size_t)b * (size_t)T + (size_t)t;
    return qkv[row * (size_t)(3 * C) + (size_t)part * (size_t)C + (size_t)h * (size_t)hs + (size_t)d];
}

/* First key position visible to query t, and last query position that sees key s. */
static inline int band_lo(int t, int window) { return t - window + 1 > 0 ? t - window + 1 : 0; }
static inline int band_hi(int s, int window, int T) { return s + window - 1 < T - 1 ? s + window - 1 : T - 1; }

/* Attention weights of one (b, h): P[t][s] for the visible band lo(t) <= s <= t,
 * 0 elsewhere, and the per-row logsumexp of the masked scaled scores.  P is a
 * T*T buffer. */
static void head_probs(const double *qkv, int T, int C, int hs, int window, int b, int h,
                       double *P, double *lse_row) {
    const double scale = 1.0 / sqrt((double)hs);
    for (int t = 0; t < T; ++t) {
        double *Pt = P + (size_t)t * (size_t)T;
        const int lo = band_lo(t, window);
        /* scores S[t][s] = q_t . k_s / sqrt(hs) for the visible s */
        double m = -INFINITY;
        for (int s = lo; s <= t; ++s) {
            double acc = 0.0;
            for (int d = 0; d < hs; ++d)
                acc += qkv_at(qkv, T, C, hs, b, t, 0, h, d) * qkv_at(qkv, T, C, hs, b, s, 1, h, d);
            Pt[s] = acc * scale;
            if (Pt[s] > m) m = Pt[s];
        }
        /* softmax over the visible row; the future (and the past outside the band) gets weight zero */
        double l = 0.0;
        for (int s = lo; s <= t; ++s) {
            Pt[s] = exp(Pt[s] - m);
            l += Pt[s];
        }
        for (int s = lo; s <= t; ++s) Pt[s] /= l;
        for (int s = 0; s < lo; ++s) Pt[s] = 0.0;
        for (int s = t + 1; s < T; ++s) Pt[s] = 0.0;
        if (lse_row) lse_row[t] = m + log(l);
    }
}

/* y[b,t,h*hs+d] = sum_s P[t][s] v_s[d] */
static void head_output(const double *qkv, int T, int C, int hs, int window, int b, int h,
                        const double *P, double *y) {
    for (int t = 0; t < T; ++t) {
        const double *Pt = P + (size_t)t * (size_t)T;
        double *yt = y + ((size_t)b * (size_t)T + (size_t)t) * (size_t)C + (size_t)h * (size_t)hs;
        for (int d = 0; d < hs; ++d) {
            double acc = 0.0;
            for (int s = band_lo(t, window); s <= t; ++s) acc += Pt[s] * qkv_at(qkv, T, C, hs, b, s, 2, h, d);
            yt[d] = acc;
        }
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Forward over a local window: y[B][T][C] and lse[B][n_head][T] (either may be
 * NULL).  window >= 1. */
int oracle_fwd_window(const double *qkv, int B, int T, int C, int n_head, int window, double *y, double *lse) {
    int rc = check_shape(B, T, C, n_head);
    if (rc) return rc;
    if (window < 1) return ORACLE_EINVAL;
    if (B == 0 || T == 0) return ORACLE_OK;
    const int hs = C / n_head;
    const int pairs = B * n_head;
    int err = 0;
#pragma omp parallel
    {
        double *P = (double *)malloc((size_t)T * (size_t)T * sizeof(double));
        if (!P) {
#pragma omp atomic write
            err = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int p = 0; p < pairs; ++p) {
            if (!P) continue;
            const int b = p / n_head, h = p % n_head;
            double *lse_row = lse ? lse + ((size_t)b * (size_t)n_head + (size_t)h) * (size_t)T : NULL;
            head_probs(qkv, T, C, hs, window, b, h, P, lse_row);
            if (y) head_output(qkv, T, C, hs, window, b, h, P, y);
        }
        free(P);
    }
    return err ? ORACLE_ENOMEM : ORACLE_OK;
}

/* Forward, causal (every past position visible). */
int oracle_fwd(const double *qkv, int B, int T, int C, int n_head, double *y, double *lse) {
    return oracle_fwd_window(qkv, B, T, C, n_head, T > 0 ? T : 1, y, lse);
}

/* Attention weights of one (b, h) as a dense T*T matrix (the "wei" of the
 * lecture's versions 2-4), for tests that inspect the weights directly. */
int oracle_probs_window(const double *qkv, int B, int T, int C, int n_head, int window, int b, int h, double *P) {
    int rc = check_shape(B, T, C, n_head);
    if (rc) return rc;
    if (window < 1 || b < 0 || b >= B || h < 0 || h >= n_head) return ORACLE_EINVAL;
    if (T == 0) return ORACLE_OK;
    head_probs(qkv, T, C, C / n_head, window, b, h, P, NULL);
    return ORACLE_OK;
}

int oracle_probs(const double *qkv, int B, int T, int C, int n_head, int b, int h, double *P) {
    return oracle_probs_window(qkv, B, T, C, n_head, T > 0 ? T : 1, b, h, P);
}

/* Backward over a local window: dqkv[B][T][3C] = d(sum y o dy)/d(qkv), by the
 * chain rule through the weighted sum, the row softmax and the scaled dot
 * products.  window >= 1. */
int oracle_bwd_window(const double *qkv, const double *dy, int B, int T, int C, int n_head, int window, double *dqkv) {
    int rc = check_shape(B, T, C, n_head);
    if (rc) return rc;
    if (window < 1) return ORACLE_EINVAL;
    if (B == 0 || T == 0) return ORACLE_OK;
    const int hs = C / n_head;
    const double scale = 1.0 / sqrt((double)hs);
    const int pairs = B * n_head;
    int err = 0;
#pragma omp parallel
    {
        double *P = (double *)malloc((size_t)T * (size_t)T * sizeof(double));
        double *dS = (double *)malloc((size_t)T * (size_t)T * sizeof(double));
        if (!P || !dS) {
#pragma omp atomic write
            err = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int p = 0; p < pairs; ++p) {
            if (!P || !dS) continue;
            const int b = p / n_head, h = p % n_head;
            head_probs(qkv, T, C, hs, window, b, h, P, NULL);
            const double *dyb = dy + (size_t)b * (size_t)T * (size_t)C + (size_t)h * (size_t)hs;
            double *dq = dqkv + (size_t)b * (size_t)T * (size_t)(3 * C) + (size_t)h * (size_t)hs;
            double *dk = dq + C;
            double *dv = dq + 2 * C;
            const size_t ld_dy = (size_t)C, ld_dqkv = (size_t)(3 * C);

            /* dP[t][s] = dy_t . v_s  (visible s only), then
             * dS[t][s] = P[t][s] * (dP[t][s] - sum_r P[t][r] dP[t][r]) */
            for (int t = 0; t < T; ++t) {
                const double *Pt = P + (size_t)t * (size_t)T;
                double *dSt = dS + (size_t)t * (size_t)T;
                const int lo = band_lo(t, window);
                double rowdot = 0.0;
                for (int s = lo; s <= t; ++s) {
                    double acc = 0.0;
                    for (int d = 0; d < hs; ++d) acc += dyb[(size_t)t * ld_dy + d] * qkv_at(qkv, T, C, hs, b, s, 2, h, d);
                    dSt[s] = acc;
                    rowdot += Pt[s] * acc;
                }
                for (int s = lo; s <= t; ++s) dSt[s] = Pt[s] * (dSt[s] - rowdot);
                for (int s = 0; s < lo; ++s) dSt[s] = 0.0;
                for (int s = t + 1; s < T; ++s) dSt[s] = 0.0;
            }
            /* dV[s] = sum over the queries t that see s of P[t][s] dy_t */
            for (int s = 0; s < T; ++s)
                for (int d = 0; d < hs; ++d) {
                    double acc = 0.0;
                    for (int t = s; t <= band_hi(s, window, T); ++t)
                        acc += P[(size_t)t * (size_t)T + s] * dyb[(size_t)t * ld_dy + d];
                    dv[(size_t)s * ld_dqkv + d] = acc;
                }
            /* dQ[t] = scale * sum over the visible s of dS[t][s] k_s */
            for (int t = 0; t < T; ++t)
                for (int d = 0; d < hs; ++d) {
                    double acc = 0.0;
                    for (int s = band_lo(t, window); s <= t; ++s)
                        acc += dS[(size_t)t * (size_t)T + s] * qkv_at(qkv, T, C, hs, b, s, 1, h, d);
                    dq[(size_t)t * ld_dqkv + d] = acc * scale;
                }
            /* dK[s] = scale * sum over the queries t that see s of dS[t][s] q_t */
            for (int s = 0; s < T; ++s)
                for (int d = 0; d < hs; ++d) {
                    double acc = 0.0;
                    for (int t = s; t <= band_hi(s, window, T); ++t)
                        acc += dS[(size_t)t * (size_t)T + s] * qkv_at(qkv, T, C, hs, b, t, 0, h, d);
                    dk[(size_t)s * ld_dqkv + d] = acc * scale;
                }
        }
        free(P);
        free(dS);
    }
    return err ? ORACLE_ENOMEM : ORACLE_OK;
}

/* Backward, causal (every past position visible). */
int oracle_bwd(const double *qkv, const double *dy, int B, int T, int C, int n_head, double *dqkv) {
    return oracle_bwd_window(qkv, dy, B, T, C, n_head, T > 0 ? T : 1, dqkv);
}
