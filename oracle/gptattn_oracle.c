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
 *  - "Let's build GPT" lecture page, chapter "scaling up the model! creating a
 *    few variables. adding dropout": dropout on the attention weights.  Read
 *    as inverted dropout after the softmax: weight P[t][s] is dropped with
 *    probability p and a kept weight is scaled by 1/(1-p); lse stays the
 *    logsumexp of the undropped scores.  The keep decision is a counter-based
 *    random number (Philox4x32-10, below), so the forward and the backward
 *    see the same mask without storing it.  p is applied in steps of 1/256:
 *    the drop probability is theta/256 with theta = round(256 p) (at most
 *    255), and kept weights are scaled by 1/(1 - theta/256).
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

/* ---------------------------------------------------------------------------
 * Philox4x32-10, written from its published definition (J. Salmon, M. Moraes,
 * R. Dror, D. Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011):
 * ten rounds on a 128-bit counter (c0, c1, c2, c3) under a 64-bit key (k0, k1).
 * A round multiplies c0 and c2 by the two round multipliers, keeps the 64-bit
 * products' high and low words, and permutes them as
 *     (hi(M1*c2) ^ c1 ^ k0,  lo(M1*c2),  hi(M0*c0) ^ c3 ^ k1,  lo(M0*c0));
 * between rounds the key is advanced by the two Weyl constants.
 * Pinned by the generator's published known-answer vectors (the Random123
 * library's list for philox4x32 with 10 rounds), besides its statistics and
 * every use of its output.
 * ------------------------------------------------------------------------- */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        const uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)c0;
        const uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)c2;
        const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
        k0 += PHILOX_W0;
        k1 += PHILOX_W1;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

/* Keep decision for attention weight (t, s) of batch-head pair bh.  One Philox
 * call covers a 4 x 4 block of (query, key) pairs: counter (s / 4, t / 4, bh, 0),
 * key = the 64-bit seed; the pair's 8 bits are byte s % 4 (least significant
 * first) of output word t % 4.  Kept iff that byte is >= theta. */
static int dropout_keep(uint64_t seed, uint32_t theta, int bh, int t, int s) {
    const uint32_t ctr[4] = {(uint32_t)s >> 2, (uint32_t)t >> 2, (uint32_t)bh, 0u};
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t r[4];
    oracle_philox4x32_10(ctr, key, r);
    return ((r[t & 3] >> (8 * (s & 3))) & 0xFFu) >= theta;
}

/* theta = round(256 p), at most 255: the drop probability is theta / 256. */
static uint32_t dropout_threshold(double p) {
    const double x = floor(256.0 * p + 0.5);
    return x >= 255.0 ? 255u : (uint32_t)x;
}

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

/* Dropout on the attention weights: p = 0 means none. */
typedef struct {
    double p;
    uint64_t seed;
} Dropout;

/* Factor applied to weight (t, s): 1/(1 - theta/256) if kept, 0 if dropped; exactly 1
 * without dropout. */
static inline double drop_factor(const Dropout *dr, int bh, int t, int s) {
    if (dr->p <= 0.0) return 1.0;
    const uint32_t theta = dropout_threshold(dr->p);
    return dropout_keep(dr->seed, theta, bh, t, s) ? 1.0 / (1.0 - theta / 256.0) : 0.0;
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

/* y[b,t,h*hs+d] = sum_s P[t][s] f[t][s] v_s[d], f the dropout factor (1 without dropout) */
static void head_output(const double *qkv, int T, int C, int hs, int window, const Dropout *dr, int n_head, int b,
                        int h, const double *P, double *y) {
    const int bh = b * n_head + h;
    for (int t = 0; t < T; ++t) {
        const double *Pt = P + (size_t)t * (size_t)T;
        double *yt = y + ((size_t)b * (size_t)T + (size_t)t) * (size_t)C + (size_t)h * (size_t)hs;
        for (int d = 0; d < hs; ++d) {
            double acc = 0.0;
            for (int s = band_lo(t, window); s <= t; ++s)
                acc += Pt[s] * drop_factor(dr, bh, t, s) * qkv_at(qkv, T, C, hs, b, s, 2, h, d);
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

/* Forward over a local window with dropout on the weights: y[B][T][C] and
 * lse[B][n_head][T] (either may be NULL).  window >= 1, 0 <= p < 1. */
int oracle_fwd_ex(const double *qkv, int B, int T, int C, int n_head, int window, double p, uint64_t seed, double *y,
                  double *lse) {
    int rc = check_shape(B, T, C, n_head);
    if (rc) return rc;
    if (window < 1 || !(p >= 0.0 && p < 1.0)) return ORACLE_EINVAL;
    const Dropout dr = {p, seed};
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
            if (y) head_output(qkv, T, C, hs, window, &dr, n_head, b, h, P, y);
        }
        free(P);
    }
    return err ? ORACLE_ENOMEM : ORACLE_OK;
}

/* Forward over a local window: y[B][T][C] and lse[B][n_head][T] (either may be
 * NULL).  window >= 1. */
int oracle_fwd_window(const double *qkv, int B, int T, int C, int n_head, int window, double *y, double *lse) {
    return oracle_fwd_ex(qkv, B, T, C, n_head, window, 0.0, 0, y, lse);
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

/* Backward over a local window with dropout on the weights: dqkv[B][T][3C] =
 * d(sum y o dy)/d(qkv) for the same dropout mask as oracle_fwd_ex, by the chain
 * rule through the weighted sum (of the dropped weights P o f), the row softmax
 * and the scaled dot products.  window >= 1, 0 <= p < 1. */
int oracle_bwd_ex(const double *qkv, const double *dy, int B, int T, int C, int n_head, int window, double p,
                  uint64_t seed, double *dqkv) {
    int rc = check_shape(B, T, C, n_head);
    if (rc) return rc;
    if (window < 1 || !(p >= 0.0 && p < 1.0)) return ORACLE_EINVAL;
    const Dropout dr = {p, seed};
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

            /* dP[t][s] = f[t][s] (dy_t . v_s)  (visible s only; dy_t . v_s is the gradient of
             * the dropped weight), then dS[t][s] = P[t][s] * (dP[t][s] - sum_r P[t][r] dP[t][r]) */
            for (int t = 0; t < T; ++t) {
                const double *Pt = P + (size_t)t * (size_t)T;
                double *dSt = dS + (size_t)t * (size_t)T;
                const int lo = band_lo(t, window);
                double rowdot = 0.0;
                for (int s = lo; s <= t; ++s) {
                    double acc = 0.0;
                    for (int d = 0; d < hs; ++d) acc += dyb[(size_t)t * ld_dy + d] * qkv_at(qkv, T, C, hs, b, s, 2, h, d);
                    acc *= drop_factor(&dr, b * n_head + h, t, s);
                    dSt[s] = acc;
                    rowdot += Pt[s] * acc;
                }
                for (int s = lo; s <= t; ++s) dSt[s] = Pt[s] * (dSt[s] - rowdot);
                for (int s = 0; s < lo; ++s) dSt[s] = 0.0;
                for (int s = t + 1; s < T; ++s) dSt[s] = 0.0;
            }
            /* dV[s] = sum over the queries t that see s of P[t][s] f[t][s] dy_t */
            for (int s = 0; s < T; ++s)
                for (int d = 0; d < hs; ++d) {
                    double acc = 0.0;
                    for (int t = s; t <= band_hi(s, window, T); ++t)
                        acc += P[(size_t)t * (size_t)T + s] * drop_factor(&dr, b * n_head + h, t, s) *
                               dyb[(size_t)t * ld_dy + d];
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

/* Backward over a local window (no dropout). */
int oracle_bwd_window(const double *qkv, const double *dy, int B, int T, int C, int n_head, int window, double *dqkv) {
    return oracle_bwd_ex(qkv, dy, B, T, C, n_head, window, 0.0, 0, dqkv);
}

/* Backward, causal (every past position visible). */
int oracle_bwd(const double *qkv, const double *dy, int B, int T, int C, int n_head, double *dqkv) {
    return oracle_bwd_window(qkv, dy, B, T, C, n_head, T > 0 ? T : 1, dqkv);
}
