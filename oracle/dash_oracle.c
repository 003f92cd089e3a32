/*
 * dash_oracle.c -- plain, slow, fp64 CPU oracle for the DashAttention forward path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * CPU-baseline leg may load this library.  It shares no code, header, table or
 * constant with the CUDA library under sparse_hierarchical_attention_stage0_b200/.
 *
 * Sources (page title, section):
 *   [S0] gist.science "DashAttention: Differentiable and Adaptive Sparse Hierarchical
 *        Attention", Technische Zusammenfassung, "Stufe 0: Lokale Chunk-Zusammenfassung"
 *        -- a learned query attends by local scaled dot-product attention over the keys
 *        of each chunk; with the query at zero this is mean pooling; a complete chunk's
 *        summary is frozen and cached.
 *   [S1] same page, "Stufe 1: Entmax-Chunk-Routing" -- w = alpha-entmax(gamma * z) over
 *        the chunk logits; GQA heads sharing a KV head share one support.
 *   [S2] same page, "Stufe 2: Prior-induzierte spaerliche Softmax" -- softmax with the
 *        reference distribution replaced by a prior g from the routing weights, g = 0
 *        where w = 0 (dynamic masking); the diagonal chunk keeps a separate branch.
 *   [E]  alpha-entmax as defined in the benchmark spec of this library:
 *        p_c = [(alpha-1) s_c - tau]_+^{1/(alpha-1)}, sum_c p_c = 1; alpha = 1 is softmax.
 *
 * Readings taken where the pages are silent (listed in the design notes):
 *   - scale 1/sqrt(D) in every stage; summaries are of the keys only;
 *   - head_cls is one vector per KV head, query head h belongs to KV head h / G;
 *   - GQA aggregation = mean of the G query heads' scores (= score of the mean query);
 *   - routable chunks of row t are the complete chunks c < floor(t / Bc);
 *   - the diagonal chunk is always attended (causal), with prior weight 1 (bias 0);
 *   - bias of an active routed chunk = sigma * log p_c.
 *
 * Every array is dense, row-major, fp64.  Layouts:
 *   Q [B,Hq,T,D], K,V [B,Hkv,T,D], head_cls [Hkv,D], summary [B,Hkv,T/Bc,D].
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double dotd(const double *a, const double *b, long n) {
    double s = 0.0;
    for (long i = 0; i < n; ++i) s += a[i] * b[i];
    return s;
}

/* ---------------------------------------------------------------- Stage 0 [S0] */

/* Summary of one chunk: softmax over the chunk's keys of hc.k_j / sqrt(D), then the
 * softmax-weighted sum of the same keys. */
static void summarize_chunk(const double *kc, long n, const double *hc, long D, double *out) {
    double *l = (double *)malloc(sizeof(double) * (size_t)n);
    double mx = -INFINITY;
    for (long j = 0; j < n; ++j) {
        l[j] = dotd(hc, kc + j * D, D) / sqrt((double)D);
        if (l[j] > mx) mx = l[j];
    }
    double den = 0.0;
    for (long j = 0; j < n; ++j) { l[j] = exp(l[j] - mx); den += l[j]; }
    for (long d = 0; d < D; ++d) out[d] = 0.0;
    for (long j = 0; j < n; ++j) {
        double w = l[j] / den;
        for (long d = 0; d < D; ++d) out[d] += w * kc[j * D + d];
    }
    free(l);
}

/* Summaries of every complete chunk: summary[b,g,c,:] for c < floor(T/Bc). */
void oracle_stage0(const double *K, const double *hc, long B, long Hkv, long T, long D,
                   long Bc, double *summary) {
    long Cf = T / Bc;
#pragma omp parallel for collapse(3) schedule(static)
    for (long b = 0; b < B; ++b)
        for (long g = 0; g < Hkv; ++g)
            for (long c = 0; c < Cf; ++c)
                summarize_chunk(K + ((b * Hkv + g) * T + c * Bc) * D, Bc, hc + g * D, D,
                                summary + ((b * Hkv + g) * Cf + c) * D);
}

/* ------------------------------------------------------------- entmax [E], [S1] */

static int cmp_desc(const void *a, const void *b) {
    double x = *(const double *)a, y = *(const double *)b;
    return (x < y) - (x > y);
}

/* f(tau) = sum_c [x_c - tau]_+^beta  (beta = 1/(alpha-1)) */
static double entmax_mass(const double *x, long n, double tau, double beta) {
    double f = 0.0;
    for (long c = 0; c < n; ++c)
        if (x[c] > tau) f += pow(x[c] - tau, beta);
    return f;
}

/* Any alpha > 1: bisection for the root of f(tau) = 1 on [max x - 1, max x - n^{1-alpha}],
 * where f(lo) >= 1 >= f(hi) and f is strictly decreasing on the bracket; 200 halvings,
 * then Newton polish steps kept inside the final bracket.  x = (alpha-1) s. */
double oracle_entmax_bisect(const double *s, long n, double alpha, double *p) {
    double beta = 1.0 / (alpha - 1.0);
    double *x = (double *)malloc(sizeof(double) * (size_t)n);
    double mx = -INFINITY;
    for (long c = 0; c < n; ++c) { x[c] = (alpha - 1.0) * s[c]; if (x[c] > mx) mx = x[c]; }
    double lo = mx - 1.0, hi = mx - pow((double)n, 1.0 - alpha);
    for (int it = 0; it < 200; ++it) {
        double mid = 0.5 * (lo + hi);
        if (entmax_mass(x, n, mid, beta) >= 1.0) lo = mid; else hi = mid;
    }
    double tau = 0.5 * (lo + hi);
    for (int it = 0; it < 4; ++it) {
        double f = -1.0, df = 0.0;
        for (long c = 0; c < n; ++c)
            if (x[c] > tau) {
                f += pow(x[c] - tau, beta);
                df += beta * pow(x[c] - tau, beta - 1.0);
            }
        if (df <= 0.0) break;
        double nt = tau + f / df;
        if (!(nt >= lo && nt <= hi)) break;
        tau = nt;
    }
    for (long c = 0; c < n; ++c) p[c] = x[c] > tau ? pow(x[c] - tau, beta) : 0.0;
    free(x);
    return tau;
}

/* alpha = 2 (sparsemax), exact: sort x descending; the support size k is the largest k
 * with 1 + k z_k > sum_{j<=k} z_j; tau = (sum_{j<=k} z_j - 1) / k
 * (Martins & Astudillo 2016, "From Softmax to Sparsemax"). */
double oracle_sparsemax_sort(const double *s, long n, double *p) {
    double *z = (double *)malloc(sizeof(double) * (size_t)n);
    for (long c = 0; c < n; ++c) z[c] = s[c];          /* alpha - 1 = 1 */
    qsort(z, (size_t)n, sizeof(double), cmp_desc);
    double cum = 0.0, tau = 0.0;
    for (long k = 1; k <= n; ++k) {
        cum += z[k - 1];
        if (1.0 + (double)k * z[k - 1] > cum) tau = (cum - 1.0) / (double)k;
    }
    for (long c = 0; c < n; ++c) p[c] = s[c] > tau ? s[c] - tau : 0.0;
    free(z);
    return tau;
}

/* alpha = 1.5, exact: sort x = s/2 descending; for the top-k set, sum (x_j - tau)^2 = 1 has
 * the root tau_k = mean_k - sqrt((1 - k * var_k) / k) (mean_k, var_k: mean and population
 * variance of the top k); the support is the largest k whose root lies below its k-th
 * value (Peters, Niculae & Martins 2019, "Sparse Sequence-to-Sequence Models"). */
double oracle_entmax15_sort(const double *s, long n, double *p) {
    double *z = (double *)malloc(sizeof(double) * (size_t)n);
    for (long c = 0; c < n; ++c) z[c] = 0.5 * s[c];
    qsort(z, (size_t)n, sizeof(double), cmp_desc);
    /* mean and M2 = k * var of the top k, updated one value at a time (Welford 1962). */
    double mean = 0.0, M2 = 0.0, tau = z[0] - 1.0;
    for (long k = 1; k <= n; ++k) {
        double dlt = z[k - 1] - mean;
        mean += dlt / (double)k;
        M2 += dlt * (z[k - 1] - mean);
        double disc = (1.0 - M2) / (double)k;
        if (disc < 0.0) break;               /* M2 never decreases: no larger support fits */
        double tk = mean - sqrt(disc);
        if (tk < z[k - 1]) tau = tk;
    }
    for (long c = 0; c < n; ++c) {
        double m = 0.5 * s[c] - tau;
        p[c] = m > 0.0 ? m * m : 0.0;
    }
    free(z);
    return tau;
}

/* alpha = 1: softmax; returns the log-sum-exp. */
double oracle_softmax(const double *s, long n, double *p) {
    double mx = -INFINITY;
    for (long c = 0; c < n; ++c) if (s[c] > mx) mx = s[c];
    double den = 0.0;
    for (long c = 0; c < n; ++c) { p[c] = exp(s[c] - mx); den += p[c]; }
    for (long c = 0; c < n; ++c) p[c] /= den;
    return mx + log(den);
}

/* Dispatch: exact sort algorithms where they exist, bisection otherwise. */
double oracle_entmax(const double *s, long n, double alpha, double *p) {
    if (alpha == 1.0) return oracle_softmax(s, n, p);
    if (alpha == 2.0) return oracle_sparsemax_sort(s, n, p);
    if (alpha == 1.5) return oracle_entmax15_sort(s, n, p);
    return oracle_entmax_bisect(s, n, alpha, p);
}

/* Top-k routing (the fixed-k block selection of the hierarchical baselines the pages compare
 * against -- liuzhao09.github.io "DashAttention 精读", sections 1-2: NSA and InfLLMv2 pick the
 * top-k blocks by coarse score, then run token-level softmax inside them): the k highest of
 * s[0..n) (ties: lower index first) are selected; p is uniform over the selection (the prior
 * of a plain softmax inside the selected blocks).  Returns theta, the k-th highest score (the
 * lowest one when k >= n). */
static int cmp_desc_idx(const void *a, const void *b) {
    const double *x = (const double *)a, *y = (const double *)b;   /* {value, index} pairs */
    if (x[0] != y[0]) return (x[0] < y[0]) - (x[0] > y[0]);
    return (x[1] > y[1]) - (x[1] < y[1]);
}

double oracle_topk(const double *s, long n, long k, double *p) {
    double *v = (double *)malloc(sizeof(double) * 2 * (size_t)n);
    for (long c = 0; c < n; ++c) { v[2 * c] = s[c]; v[2 * c + 1] = (double)c; p[c] = 0.0; }
    qsort(v, (size_t)n, 2 * sizeof(double), cmp_desc_idx);
    long ke = k < n ? k : n;
    for (long i = 0; i < ke; ++i) p[(long)v[2 * i + 1]] = 1.0 / (double)ke;
    double theta = v[2 * (ke - 1)];
    free(v);
    return theta;
}

/* ---------------------------------------------------------------- Stage 1 [S1] */

/* Routing of one row from its group-mean query qbar over the ct routable chunks S[0..ct).
 * With dsum non-NULL (estimate_diagonal) the diagonal chunk ct takes part in the alpha-entmax
 * normalisation as one more candidate, its score taken against the estimated summary dsum
 * (aiexpert.news interface paragraph: estimate_diagonal is the diagonal correction of the
 * alpha-entmax normalisation; gist.science "Stufe 2": chunks near the diagonal may have no
 * summary).  With topk > 0 the routing is the top-k selection of oracle_topk instead of
 * alpha-entmax.  p_row, m_row have C entries: p_c and the margin m_c = (alpha-1) s_c - tau for
 * the routed candidates (margin +inf for alpha = 1; s_c - theta for top-k), p = 0 and m = NaN
 * elsewhere.  Returns tau (the log-sum-exp for alpha = 1; theta for top-k; NaN when there is
 * no candidate). */
static double route_qbar(const double *qbar, const double *S, long ct, long C, long D,
                         double alpha, double gamma, const double *dsum, long topk,
                         double *p_row, double *m_row) {
    for (long c = 0; c < C; ++c) { p_row[c] = 0.0; m_row[c] = NAN; }
    long n = ct + (dsum ? 1 : 0);
    if (n == 0) return NAN;
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    for (long c = 0; c < ct; ++c)
        s[c] = gamma * dotd(qbar, S + c * D, D) / sqrt((double)D);
    if (dsum) s[ct] = gamma * dotd(qbar, dsum, D) / sqrt((double)D);
    double tau;
    if (topk > 0) {                      /* margins s - theta: >= 0 on the selection */
        tau = oracle_topk(s, n, topk, p_row);
        for (long c = 0; c < n; ++c) m_row[c] = s[c] - tau;
    } else {
        tau = oracle_entmax(s, n, alpha, p_row);
        for (long c = 0; c < n; ++c)
            m_row[c] = alpha == 1.0 ? INFINITY : (alpha - 1.0) * s[c] - tau;
    }
    free(s);
    return tau;
}

/* Estimated summary of the diagonal chunk of row t: Stage 0's softmax-weighted key sum over
 * the keys of chunk ct = t / Bc that the row can see (ct Bc .. t). */
static void diag_summary(const double *Kg, long t, long Bc, const double *hc, long D,
                         double *out) {
    long ct = t / Bc;
    summarize_chunk(Kg + ct * Bc * D, t - ct * Bc + 1, hc, D, out);
}

/* Group-mean query of KV group g: the mean of the G query rows q_h, h in [gG, (g+1)G).
 * Averaging the G heads' scores equals scoring this mean query (linearity). */
static void group_mean(const double *q0, long stride, long G, long D, double *qbar) {
    for (long d = 0; d < D; ++d) qbar[d] = 0.0;
    for (long h = 0; h < G; ++h)
        for (long d = 0; d < D; ++d) qbar[d] += q0[h * stride + d];
    for (long d = 0; d < D; ++d) qbar[d] /= (double)G;
}

/* Stage 1 for a list of rows, with K [B,Hkv,T,D] and head_cls non-NULL when estimating the
 * diagonal chunk's score, and topk > 0 for top-k routing (see route_qbar); outputs as
 * oracle_stage1. */
void oracle_stage1_diag(const double *Q, const double *summary, const double *K,
                        const double *hc, long B, long Hq, long Hkv, long T, long D, long Bc,
                        double alpha, double gamma, long topk, const int64_t *rows, long nrows,
                        double *p_out, double *m_out, double *tau_out) {
    long G = Hq / Hkv, Cf = T / Bc, C = (T + Bc - 1) / Bc;
#pragma omp parallel for collapse(3) schedule(dynamic, 16)
    for (long b = 0; b < B; ++b)
        for (long g = 0; g < Hkv; ++g)
            for (long r = 0; r < nrows; ++r) {
                long o = (b * Hkv + g) * nrows + r, t = rows[r];
                double *qbar = (double *)malloc(sizeof(double) * (size_t)D);
                double *dsum = NULL;
                group_mean(Q + ((b * Hq + g * G) * T + t) * D, T * D, G, D, qbar);
                if (K) {
                    dsum = (double *)malloc(sizeof(double) * (size_t)D);
                    diag_summary(K + (b * Hkv + g) * T * D, t, Bc, hc + g * D, D, dsum);
                }
                tau_out[o] = route_qbar(qbar, summary + (b * Hkv + g) * Cf * D, t / Bc, C, D,
                                        alpha, gamma, dsum, topk, p_out + o * C, m_out + o * C);
                free(dsum);
                free(qbar);
            }
}

/* Stage 1 for a list of rows.  summary is [B,Hkv,T/Bc,D] (T is the sequence length the
 * summaries were built from).  Outputs: p_out, m_out [B,Hkv,nrows,C], tau_out [B,Hkv,nrows],
 * with C = ceil(T/Bc). */
void oracle_stage1(const double *Q, const double *summary, long B, long Hq, long Hkv, long T,
                   long D, long Bc, double alpha, double gamma, const int64_t *rows,
                   long nrows, double *p_out, double *m_out, double *tau_out) {
    oracle_stage1_diag(Q, summary, NULL, NULL, B, Hq, Hkv, T, D, Bc, alpha, gamma, 0, rows,
                       nrows, p_out, m_out, tau_out);
}

/* ---------------------------------------------------------------- Stage 2 [S2] */

/* One (b, h, t) output row.  Keys j <= t; key j of chunk c = j / Bc gets
 *   bias 0               if c == ct (diagonal branch) or dense != 0,
 *   bias sigma * log p_c if c < ct and p_c > 0,
 *   no weight at all     if c < ct and p_c == 0 (dynamic masking).
 * out = sum_j softmax_j(q.k_j / sqrt(D) + bias_j) v_j, with the exact maximum. */
static void attend_row(const double *q, const double *Kg, const double *Vg, const double *p_row,
                       long t, long D, long Bc, double sigma, int dense, double *out) {
    long ct = t / Bc, n = t + 1;
    double *l = (double *)malloc(sizeof(double) * (size_t)n);
    double mx = -INFINITY;
    for (long j = 0; j < n; ++j) {
        long c = j / Bc;
        if (c == ct || dense) {
            l[j] = dotd(q, Kg + j * D, D) / sqrt((double)D);
        } else if (p_row[c] > 0.0) {
            l[j] = dotd(q, Kg + j * D, D) / sqrt((double)D) + sigma * log(p_row[c]);
        } else {
            l[j] = -INFINITY;
        }
        if (l[j] > mx) mx = l[j];
    }
    double den = 0.0;
    for (long d = 0; d < D; ++d) out[d] = 0.0;
    for (long j = 0; j < n; ++j) {
        if (l[j] == -INFINITY) continue;
        double w = exp(l[j] - mx);
        den += w;
        for (long d = 0; d < D; ++d) out[d] += w * Vg[j * D + d];
    }
    for (long d = 0; d < D; ++d) out[d] /= den;
    free(l);
}

/* Stage 2 for a list of rows.  p is [B,Hkv,nrows,C] (the routing of the same rows) or NULL
 * when dense != 0.  O_out is [B,Hq,nrows,D]. */
void oracle_stage2(const double *Q, const double *K, const double *V, const double *p, long B,
                   long Hq, long Hkv, long T, long D, long Bc, double sigma, int dense,
                   const int64_t *rows, long nrows, double *O_out) {
    long G = Hq / Hkv, C = (T + Bc - 1) / Bc;
#pragma omp parallel for collapse(3) schedule(dynamic, 4)
    for (long b = 0; b < B; ++b)
        for (long h = 0; h < Hq; ++h)
            for (long r = 0; r < nrows; ++r) {
                long g = h / G, t = rows[r];
                const double *prow = p ? p + ((b * Hkv + g) * nrows + r) * C : NULL;
                attend_row(Q + ((b * Hq + h) * T + t) * D, K + (b * Hkv + g) * T * D,
                           V + (b * Hkv + g) * T * D, prow, t, D, Bc, sigma, dense,
                           O_out + ((b * Hq + h) * nrows + r) * D);
            }
}

/* ---------------------------------------------------------------- decode */

/* One incremental-decode step for B independent sequences.  Caches K,V [B,Hkv,cap,D] hold
 * seq_lens[b] valid tokens (the current token included); q is [B,Hq,D] for the token at
 * t = seq_lens[b]-1.  The chunk summaries of the complete chunks are recomputed here from
 * the cache keys (the frozen cache of [S0] holds exactly these values).  Outputs:
 * O [B,Hq,D], p and m [B,Hkv,Ccap] (Ccap = ceil(cap/Bc)), tau [B,Hkv]. */
void oracle_decode(const double *q, const double *K, const double *V, const double *hc,
                   const int64_t *seq_lens, long B, long Hq, long Hkv, long cap, long D,
                   long Bc, double alpha, double gamma, double sigma, int estimate_diagonal,
                   long topk, double *O, double *p, double *m, double *tau) {
    long G = Hq / Hkv, Ccap = (cap + Bc - 1) / Bc;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (long b = 0; b < B; ++b)
        for (long g = 0; g < Hkv; ++g) {
            long L = seq_lens[b], t = L - 1, ct = t / Bc;
            const double *Kg = K + (b * Hkv + g) * cap * D;
            const double *Vg = V + (b * Hkv + g) * cap * D;
            double *S = (double *)malloc(sizeof(double) * (size_t)((ct > 0 ? ct : 1) * D));
            for (long c = 0; c < ct; ++c)
                summarize_chunk(Kg + c * Bc * D, Bc, hc + g * D, D, S + c * D);
            double *pr = p + (b * Hkv + g) * Ccap, *mr = m + (b * Hkv + g) * Ccap;
            double *qbar = (double *)malloc(sizeof(double) * (size_t)D);
            group_mean(q + (b * Hq + g * G) * D, D, G, D, qbar);
            double *dsum = NULL;
            if (estimate_diagonal) {
                dsum = (double *)malloc(sizeof(double) * (size_t)D);
                diag_summary(Kg, t, Bc, hc + g * D, D, dsum);
            }
            double tv = route_qbar(qbar, S, ct, Ccap, D, alpha, gamma, dsum, topk, pr, mr);
            free(dsum);
            free(qbar);
            tau[b * Hkv + g] = tv;
            for (long h = g * G; h < (g + 1) * G; ++h)
                attend_row(q + (b * Hq + h) * D, Kg, Vg, pr, t, D, Bc, sigma, 0,
                           O + (b * Hq + h) * D);
            free(S);
        }
}

/* Routing alone of one decode step (liuzhao09.github.io "DashAttention 精读" section 2:
 * incremental decoding reuses the cached chunk representations; gist.science summary,
 * "Stufe 0": a complete chunk's summary is frozen).  For each sequence b the query row is
 * t = seq_lens[b]-1, routed over its complete chunks c < t / Bc from the given summaries
 * [B,Hkv,Cs,D] (any Cs > t / Bc - 1): the Stage 1 routing of that row.  q is [B,Hq,D].  With
 * the key cache K [B,Hkv,cap,D] and head_cls non-NULL the diagonal chunk's score is estimated
 * too (see route_qbar).  Outputs: p and m [B,Hkv,Ccap], Ccap = ceil(cap/Bc), tau [B,Hkv] (as
 * oracle_decode). */
void oracle_decode_route(const double *q, const double *summary, const double *K,
                         const double *hc, const int64_t *seq_lens, long B, long Hq, long Hkv,
                         long Cs, long cap, long D, long Bc, double alpha, double gamma,
                         long topk, double *p, double *m, double *tau) {
    long Ccap = (cap + Bc - 1) / Bc;
    long G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (long b = 0; b < B; ++b)
        for (long g = 0; g < Hkv; ++g) {
            long t = seq_lens[b] - 1, ct = t / Bc;
            double *qbar = (double *)malloc(sizeof(double) * (size_t)D);
            double *dsum = NULL;
            group_mean(q + (b * Hq + g * G) * D, D, G, D, qbar);
            if (K) {
                dsum = (double *)malloc(sizeof(double) * (size_t)D);
                diag_summary(K + (b * Hkv + g) * cap * D, t, Bc, hc + g * D, D, dsum);
            }
            tau[b * Hkv + g] = route_qbar(qbar, summary + (b * Hkv + g) * Cs * D, ct, Ccap, D,
                                          alpha, gamma, dsum, topk, p + (b * Hkv + g) * Ccap,
                                          m + (b * Hkv + g) * Ccap);
            free(dsum);
            free(qbar);
        }
}

/* ---------------------------------------------------------------- backward */

/* Gradients of L = sum(O * dO) with respect to Q, K, V and head_cls, through all three stages
 * (gist.science summary, "Stufe 1": alpha-entmax is differentiable, so gradients flow from the
 * Stage 2 softmax through the routing back to the chunk summaries of Stage 0;
 * liuzhao09.github.io "DashAttention 精读", section 2: the hierarchy trains end to end).
 * Written from the chain rule of the forward above, one stage at a time (prefill, default
 * mode: entmax routing, bias sigma * log p on routed chunks, diagonal with bias 0):
 *   Stage 2, row (h, t), attention weights a_j over its attended keys, O = sum a_j v_j:
 *     dl_j = a_j (dO . v_j - dO . O);  dq += sum_j dl_j k_j / sqrt(D);  dk_j += dl_j q / sqrt(D);
 *     dv_j += a_j dO;  a routed chunk c (p_c > 0) collects dlogp_c += sigma * sum_{j in c} dl_j.
 *   Routing, row (g, t): dp_c = dlogp_c / p_c on the support; with g_c = p_c^(2 - alpha)
 *     (p_c for alpha = 1) the entmax Jacobian (Peters, Niculae & Martins 2019) gives
 *     ds_c = g_c dp_c - g_c (sum g dp) / (sum g);  s_c = gamma qbar . S_c / sqrt(D), so
 *     dqbar = sum_c ds_c gamma S_c / sqrt(D) (each of the G heads gets dqbar / G) and
 *     dS_c += ds_c gamma qbar / sqrt(D).
 *   Stage 0, chunk c with weights w = softmax(hc . k_j / sqrt(D)), S_c = sum w_j k_j:
 *     dk_j += w_j dS_c;  dl_j = w_j (k_j . dS_c - S_c . dS_c);  dk_j += dl_j hc / sqrt(D);
 *     dhc += dl_j k_j / sqrt(D).
 * Outputs are overwritten; dhc [Hkv, D] sums over the batch. */
void oracle_backward(const double *Q, const double *K, const double *V, const double *hc,
                     const double *dO, long B, long Hq, long Hkv, long T, long D, long Bc,
                     double alpha, double gamma, double sigma, double *dQ, double *dK,
                     double *dV, double *dhc) {
    long G = Hq / Hkv, Cf = T / Bc, C = (T + Bc - 1) / Bc;
    double rs = 1.0 / sqrt((double)D);
    for (long i = 0; i < B * Hq * T * D; ++i) dQ[i] = 0.0;
    for (long i = 0; i < B * Hkv * T * D; ++i) { dK[i] = 0.0; dV[i] = 0.0; }
    double *dhc_bg = (double *)calloc((size_t)(B * Hkv * D), sizeof(double));
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (long b = 0; b < B; ++b)
        for (long g = 0; g < Hkv; ++g) {
            const double *Kg = K + (b * Hkv + g) * T * D, *Vg = V + (b * Hkv + g) * T * D;
            double *dKg = dK + (b * Hkv + g) * T * D, *dVg = dV + (b * Hkv + g) * T * D;
            const double *hcg = hc + g * D;
            /* forward: summaries */
            double *S = (double *)calloc((size_t)((Cf > 0 ? Cf : 1) * D), sizeof(double));
            double *dS = (double *)calloc((size_t)((Cf > 0 ? Cf : 1) * D), sizeof(double));
            for (long c = 0; c < Cf; ++c) summarize_chunk(Kg + c * Bc * D, Bc, hcg, D, S + c * D);
            double *qbar = (double *)malloc(sizeof(double) * (size_t)D);
            double *pr = (double *)malloc(sizeof(double) * (size_t)C);
            double *mr = (double *)malloc(sizeof(double) * (size_t)C);
            double *dlogp = (double *)malloc(sizeof(double) * (size_t)C);
            double *l = (double *)malloc(sizeof(double) * (size_t)T);
            double *O = (double *)malloc(sizeof(double) * (size_t)D);
            for (long t = 0; t < T; ++t) {
                long ct = t / Bc, n = t + 1;
                group_mean(Q + ((b * Hq + g * G) * T + t) * D, T * D, G, D, qbar);
                route_qbar(qbar, S, ct, C, D, alpha, gamma, NULL, 0, pr, mr);
                for (long c = 0; c < C; ++c) dlogp[c] = 0.0;
                for (long h = g * G; h < (g + 1) * G; ++h) {
                    const double *q = Q + ((b * Hq + h) * T + t) * D;
                    const double *dOr = dO + ((b * Hq + h) * T + t) * D;
                    double *dq = dQ + ((b * Hq + h) * T + t) * D;
                    /* forward row: logits, weights (exact maximum), O */
                    double mx = -INFINITY;
                    for (long j = 0; j < n; ++j) {
                        long c = j / Bc;
                        if (c == ct) l[j] = dotd(q, Kg + j * D, D) * rs;
                        else if (pr[c] > 0.0) l[j] = dotd(q, Kg + j * D, D) * rs + sigma * log(pr[c]);
                        else l[j] = -INFINITY;
                        if (l[j] > mx) mx = l[j];
                    }
                    double den = 0.0;
                    for (long j = 0; j < n; ++j) { l[j] = l[j] == -INFINITY ? 0.0 : exp(l[j] - mx); den += l[j]; }
                    for (long d = 0; d < D; ++d) O[d] = 0.0;
                    for (long j = 0; j < n; ++j) {
                        l[j] /= den;                                /* l now holds a_j */
                        for (long d = 0; d < D; ++d) O[d] += l[j] * Vg[j * D + d];
                    }
                    double dOO = dotd(dOr, O, D);
                    for (long j = 0; j < n; ++j) {
                        if (l[j] == 0.0) continue;
                        double dl = l[j] * (dotd(dOr, Vg + j * D, D) - dOO);
                        for (long d = 0; d < D; ++d) {
                            dq[d] += dl * Kg[j * D + d] * rs;
                            dKg[j * D + d] += dl * q[d] * rs;
                            dVg[j * D + d] += l[j] * dOr[d];
                        }
                        long c = j / Bc;
                        if (c < ct) dlogp[c] += sigma * dl;
                    }
                }
                if (ct == 0) continue;
                /* routing backward: entmax Jacobian on the support */
                double sg = 0.0, sgdp = 0.0;
                for (long c = 0; c < ct; ++c) {
                    if (!(pr[c] > 0.0)) continue;
                    double gc = alpha == 1.0 ? pr[c] : pow(pr[c], 2.0 - alpha);
                    sg += gc;
                    sgdp += gc * dlogp[c] / pr[c];
                }
                for (long c = 0; c < ct; ++c) {
                    if (!(pr[c] > 0.0)) continue;
                    double gc = alpha == 1.0 ? pr[c] : pow(pr[c], 2.0 - alpha);
                    double ds = gc * dlogp[c] / pr[c] - gc * sgdp / sg;
                    for (long d = 0; d < D; ++d) {
                        double dqb = ds * gamma * S[c * D + d] * rs;
                        for (long h = g * G; h < (g + 1) * G; ++h)
                            dQ[((b * Hq + h) * T + t) * D + d] += dqb / (double)G;
                        dS[c * D + d] += ds * gamma * qbar[d] * rs;
                    }
                }
            }
            /* Stage 0 backward */
            double *w = (double *)malloc(sizeof(double) * (size_t)Bc);
            for (long c = 0; c < Cf; ++c) {
                const double *kc = Kg + c * Bc * D;
                double mx = -INFINITY, den = 0.0, sdS = dotd(S + c * D, dS + c * D, D);
                for (long j = 0; j < Bc; ++j) { w[j] = dotd(hcg, kc + j * D, D) * rs; if (w[j] > mx) mx = w[j]; }
                for (long j = 0; j < Bc; ++j) { w[j] = exp(w[j] - mx); den += w[j]; }
                for (long j = 0; j < Bc; ++j) {
                    w[j] /= den;
                    double dl = w[j] * (dotd(kc + j * D, dS + c * D, D) - sdS);
                    for (long d = 0; d < D; ++d) {
                        dKg[(c * Bc + j) * D + d] += w[j] * dS[c * D + d] + dl * hcg[d] * rs;
                        dhc_bg[(b * Hkv + g) * D + d] += dl * kc[j * D + d] * rs;
                    }
                }
            }
            free(w); free(S); free(dS); free(qbar); free(pr); free(mr); free(dlogp); free(l); free(O);
        }
    for (long g = 0; g < Hkv; ++g)
        for (long d = 0; d < D; ++d) {
            double acc = 0.0;
            for (long b = 0; b < B; ++b) acc += dhc_bg[(b * Hkv + g) * D + d];
            dhc[g * D + d] = acc;
        }
    free(dhc_bg);
}

/* Number of OpenMP threads the oracle runs with (for reporting). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
