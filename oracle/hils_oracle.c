/*
 * HiLS-Attention oracle: a plain, slow, fp64 CPU statement of what the hot path computes.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call this file;
 * only the test-suite, the smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * Source: "Hierarchical Sparse Attention Done Right: Toward Infinite Context Modeling"
 * (arXiv 2607.02980). Citations name the page section / equation they follow:
 *   - Sec. 2 (BSA preliminaries): chunk partition, chunk-aligned sliding window, candidate set.
 *   - Sec. 3 RQ1, Prop. 3.1, Eq. 7 and Eq. 8: landmark summary k'_c, entropy bias b'_c and the
 *     retrieval score s^_{i,c} = q^_i.k'_c / sqrt(d) + b'_c.
 *   - Sec. 4 "GQA": per-head normalised chunk weights, max over the heads of a group, shared top-k.
 *   - Sec. 3 RQ2 and the picx.dev summary's Eq. 10: hierarchical softmax
 *     w_ij = exp(s_ij)/Z_{i,c(j)} * Z^_{i,c(j)}/Z^_i, Z^_i normalising over selected chunks + window.
 *
 * Readings where the pages are silent (all listed with reasons in the design notes):
 *   window  : left edge l_p = S*floor(max(0, p-W+1)/S); window tokens [l_p, p];
 *             candidates are chunks c < l_p/S (all complete and wholly left of the window).
 *   GQA     : per-head log-softmax of s^ over the candidates only; group score = max over heads;
 *             top-min(k, n_p) by (score desc, chunk id asc); idx rows ascending, -1 padded.
 *   window in Z^: the window keeps its exact mass sum_j exp(s_ij) (its raw logits).
 *   idx as a set: entries outside [0, n_p) are ignored, a repeated id counts once.
 *   scale   : tau (default 1/sqrt(d)) for token, landmark and retrieval logits alike.
 *
 * Parity status per function is stated above each one ("pinned by" = the independent facts the
 * tests check it against).
 *
 * Layouts (row-major, contiguous, fp64):
 *   q, q_hat [B,Hq,T,d]   k, v [B,Hkv,L,d]   q_land, k_sum [B,Hq,Nc,d]   b_sum [B,Hq,Nc]
 *   idx [B,Hkv,T,topk] int32   gap [B,Hkv,T]   out, dout [B,Hq,T,d]   lse [B,Hq,T]
 * with Nc = floor(L/S), G = Hq/Hkv, head h reads KV head h/G, query row i sits at position q_pos0+i.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int B, T, L, Hq, Hkv, d, S, topk, W, q_pos0;
    double scale; /* <= 0 means 1/sqrt(d) */
} orc_params;

static double tau_of(const orc_params *p) { return p->scale > 0 ? p->scale : 1.0 / sqrt((double)p->d); }

static double dot(const double *a, const double *b, int n) {
    double s = 0.0;
    for (int t = 0; t < n; ++t) s += a[t] * b[t];
    return s;
}

/* log(sum_t exp(x_t)) with the maximum subtracted first; -inf for n == 0. */
static double logsumexp(const double *x, int n) {
    if (n <= 0) return -INFINITY;
    double m = x[0];
    for (int t = 1; t < n; ++t) if (x[t] > m) m = x[t];
    if (m == -INFINITY) return -INFINITY;
    double s = 0.0;
    for (int t = 0; t < n; ++t) s += exp(x[t] - m);
    return m + log(s);
}

/* Sec. 2: aligned window left edge for absolute position pos. */
static int window_left(const orc_params *p, int pos) {
    int e = pos - p->W + 1;
    if (e < 0) e = 0;
    return (e / p->S) * p->S;
}

void orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int orc_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Sec. 2 window + candidate count for every query row (exported so tests can pin the reading). */
void orc_window(const orc_params *p, int *left, int *n_cand) {
    for (int i = 0; i < p->T; ++i) {
        int pos = p->q_pos0 + i;
        left[i] = window_left(p, pos);
        n_cand[i] = left[i] / p->S;
    }
}

/*
 * Eq. 8 (Prop. 3.1): for every batch b, query head h and complete chunk c in [c_begin, c_end):
 *   u_j = tau * q'_{h,c} . k_j  (j in chunk c, KV head h/G),  p = softmax(u),
 *   k'_{h,c} = sum_j p_j k_j,   b'_{h,c} = -sum_j p_j log p_j.
 * Pinned by: S = 1 (k' = k, b' = 0), uniform logits (k' = mean key, b' = log S), the two-token
 * closed form (binary entropy), and the Eq. 7 tangency / lower-bound facts.
 */
void orc_chunk_summary(const orc_params *p, const double *k, const double *q_land, int c_begin, int c_end,
                       double *k_sum, double *b_sum) {
    const int d = p->d, S = p->S, G = p->Hq / p->Hkv, Nc = p->L / p->S;
    const double tau = tau_of(p);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < p->B; ++b)
        for (int h = 0; h < p->Hq; ++h) {
            double *u = (double *)malloc(sizeof(double) * S);
            const double *kh = k + ((size_t)b * p->Hkv + h / G) * (size_t)p->L * d;
            for (int c = c_begin; c < c_end; ++c) {
                const double *ql = q_land + (((size_t)b * p->Hq + h) * Nc + c) * d;
                for (int j = 0; j < S; ++j) u[j] = tau * dot(ql, kh + (size_t)(c * S + j) * d, d);
                double lse = logsumexp(u, S);
                double *ks = k_sum + (((size_t)b * p->Hq + h) * Nc + c) * d;
                for (int t = 0; t < d; ++t) ks[t] = 0.0;
                double ent = 0.0;
                for (int j = 0; j < S; ++j) {
                    double logp = u[j] - lse;
                    double pj = exp(logp);
                    for (int t = 0; t < d; ++t) ks[t] += pj * kh[(size_t)(c * S + j) * d + t];
                    ent -= pj * logp;
                }
                b_sum[((size_t)b * p->Hq + h) * Nc + c] = ent;
            }
            free(u);
        }
}

/* Eq. 7 / Eq. 10 retrieval score s^_{h,c} for query vector qh (length d). */
static double retrieval_score(const orc_params *p, const double *qh, const double *k_sum, const double *b_sum,
                              int b, int h, int c) {
    const int Nc = p->L / p->S;
    const size_t row = ((size_t)b * p->Hq + h) * Nc + c;
    return tau_of(p) * dot(qh, k_sum + row * p->d, p->d) + b_sum[row];
}

typedef struct { double g; int c; } cand_t;

static int cand_cmp(const void *x, const void *y) {
    const cand_t *a = (const cand_t *)x, *b = (const cand_t *)y;
    if (a->g > b->g) return -1;
    if (a->g < b->g) return 1;
    return (a->c < b->c) ? -1 : (a->c > b->c);
}

static int int_cmp(const void *x, const void *y) {
    int a = *(const int *)x, b = *(const int *)y;
    return (a > b) - (a < b);
}

/*
 * Sec. 4 "GQA" selection from per-head chunk scores sc[hh*n + c] (hh < G, c < n) of one (b, g, row):
 *   per-head log-normalised weight sc_{h,c} - LSE_{c'<n} sc_{h,c'}; group score g_c = max over heads;
 *   keep min(topk, n) candidates by (g desc, c asc); write them ascending, pad with -1.
 * gap (nullable) = g_(topk) - g_(topk+1) in the sorted order, +inf when n <= topk.
 */
static void group_topk(int G, int n, int K, const double *sc, int *out, double *gp) {
    for (int t = 0; t < K; ++t) out[t] = -1;
    if (n == 0) {
        if (gp) *gp = INFINITY;
        return;
    }
    cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * n);
    for (int c = 0; c < n; ++c) { cand[c].g = -INFINITY; cand[c].c = c; }
    for (int hh = 0; hh < G; ++hh) {
        const double z = logsumexp(sc + (size_t)hh * n, n);
        for (int c = 0; c < n; ++c) {
            double w = sc[(size_t)hh * n + c] - z;
            if (w > cand[c].g) cand[c].g = w;
        }
    }
    qsort(cand, n, sizeof(cand_t), cand_cmp);
    const int kk = n < K ? n : K;
    for (int t = 0; t < kk; ++t) out[t] = cand[t].c;
    qsort(out, kk, sizeof(int), int_cmp);
    if (gp) *gp = (n > K) ? cand[K - 1].g - cand[K].g : INFINITY;
    free(cand);
}

/*
 * Sec. 3 RQ1 (top-k over the retrieval scores) with Sec. 4 "GQA": for every (b, KV group g, row i)
 * at position pos with n candidates, s^_{h,c} for c < n and every head h of the group, then the
 * group selection above.
 * Pinned by: planted dominant chunks, tie rule on identical chunks, per-head shift invariance,
 * G = 1 reduction (top-k of raw s^), and the naive-BSA special case.
 */
void orc_select_topk(const orc_params *p, const double *q_hat, const double *k_sum, const double *b_sum, int *idx,
                     double *gap) {
    const int G = p->Hq / p->Hkv, K = p->topk;
#pragma omp parallel for collapse(3) schedule(dynamic)
    for (int b = 0; b < p->B; ++b)
        for (int g = 0; g < p->Hkv; ++g)
            for (int i = 0; i < p->T; ++i) {
                const int pos = p->q_pos0 + i;
                const int n = window_left(p, pos) / p->S;
                int *out = idx + (((size_t)b * p->Hkv + g) * p->T + i) * K;
                double *gp = gap ? gap + ((size_t)b * p->Hkv + g) * p->T + i : NULL;
                double *sh = (double *)malloc(sizeof(double) * ((size_t)G * n + 1));
                for (int hh = 0; hh < G; ++hh) {
                    const int h = g * G + hh;
                    const double *qh = q_hat + (((size_t)b * p->Hq + h) * p->T + i) * p->d;
                    for (int c = 0; c < n; ++c) sh[(size_t)hh * n + c] = retrieval_score(p, qh, k_sum, b_sum, b, h, c);
                }
                group_topk(G, n, K, sh, out, gp);
                free(sh);
            }
}

/*
 * Naive BSA (Sec. 2): the exact chunk mass of candidate c for row i under head h is
 * sum_{j in c} exp(s_ij), s_ij = tau q_i.k_j; its log, M_{h,c} = LSE_{j in c} s_ij, takes the place of
 * s^ in the same group selection (per-head normalisation over the candidates, max over the group's
 * heads, top-k by (score desc, id asc)). mass (nullable) [B,Hq,T,Nc]: M_{h,c} for c < n, entries
 * c >= n left untouched. With G = 1 this is top-k by raw chunk mass, the rule Sec. 2 states.
 * Pinned by: brute-force chunk masses and top-k on tiny inputs, equality with the HiLS selection on
 * chunk-constant keys (where the summary is exact, Prop. 3.1), and a planted two-head GQA case.
 */
void orc_bsa_select_topk(const orc_params *p, const double *q, const double *k, int *idx, double *gap,
                         double *mass) {
    const int G = p->Hq / p->Hkv, K = p->topk, S = p->S, d = p->d, Nc = p->L / p->S;
    const double tau = tau_of(p);
#pragma omp parallel for collapse(3) schedule(dynamic)
    for (int b = 0; b < p->B; ++b)
        for (int g = 0; g < p->Hkv; ++g)
            for (int i = 0; i < p->T; ++i) {
                const int pos = p->q_pos0 + i;
                const int n = window_left(p, pos) / S;
                int *out = idx + (((size_t)b * p->Hkv + g) * p->T + i) * K;
                double *gp = gap ? gap + ((size_t)b * p->Hkv + g) * p->T + i : NULL;
                double *m = (double *)malloc(sizeof(double) * ((size_t)G * n + 1));
                double *s = (double *)malloc(sizeof(double) * S);
                for (int hh = 0; hh < G; ++hh) {
                    const int h = g * G + hh;
                    const double *qi = q + (((size_t)b * p->Hq + h) * p->T + i) * d;
                    for (int c = 0; c < n; ++c) {
                        for (int j = 0; j < S; ++j)
                            s[j] = tau * dot(qi, k + (((size_t)b * p->Hkv + g) * p->L + (size_t)c * S + j) * d, d);
                        m[(size_t)hh * n + c] = logsumexp(s, S);
                        if (mass) mass[(((size_t)b * p->Hq + h) * p->T + i) * Nc + c] = m[(size_t)hh * n + c];
                    }
                }
                group_topk(G, n, K, m, out, gp);
                free(s);
                free(m);
            }
}

/* The valid, distinct chunk ids of one idx row, ascending; returns their count. */
static int selected_set(const int *row, int K, int n_cand, int *sel) {
    int m = 0;
    for (int t = 0; t < K; ++t) {
        int c = row[t];
        if (c < 0 || c >= n_cand) continue;
        int dup = 0;
        for (int u = 0; u < m; ++u) if (sel[u] == c) dup = 1;
        if (!dup) sel[m++] = c;
    }
    qsort(sel, m, sizeof(int), int_cmp);
    return m;
}

/*
 * Sec. 3 RQ2, Eq. 10 in chunked form, for every (b, h, row i) at position pos:
 *   window tokens j in [l, pos]: raw logits s_j = tau q.k_j;
 *   for each selected chunk c: s^_c (Eq. 7), L_c = LSE_{j in c} s_j, o_c = sum_j exp(s_j - L_c) v_j;
 *   log Z^ = LSE({s_j}_window U {s^_c}_selected);
 *   out = sum_window exp(s_j - log Z^) v_j + sum_c exp(s^_c - log Z^) o_c,  lse = log Z^.
 * Pinned by: weights summing to one (v = 1 gives out = 1), the token-by-token Eq. 10 evaluation,
 * exact causal softmax attention on chunk-constant keys with everything selected, sliding-window
 * attention when no chunk is a candidate, idx permutation invariance, and MHA = GQA with G = 1.
 */
void orc_attn_fwd(const orc_params *p, const double *q, const double *k, const double *v, const double *q_hat,
                  const double *k_sum, const double *b_sum, const int *idx, double *out, double *lse) {
    const int d = p->d, S = p->S, G = p->Hq / p->Hkv, K = p->topk;
    const double tau = tau_of(p);
#pragma omp parallel for collapse(3) schedule(dynamic)
    for (int b = 0; b < p->B; ++b)
        for (int h = 0; h < p->Hq; ++h)
            for (int i = 0; i < p->T; ++i) {
                const int g = h / G, pos = p->q_pos0 + i;
                const int l = window_left(p, pos), n = l / S;
                const double *qi = q + (((size_t)b * p->Hq + h) * p->T + i) * d;
                const double *qhi = q_hat + (((size_t)b * p->Hq + h) * p->T + i) * d;
                const double *kb = k + ((size_t)b * p->Hkv + g) * (size_t)p->L * d;
                const double *vb = v + ((size_t)b * p->Hkv + g) * (size_t)p->L * d;
                int *sel = (int *)malloc(sizeof(int) * (K > 0 ? K : 1));
                const int m = selected_set(idx + (((size_t)b * p->Hkv + g) * p->T + i) * K, K, n, sel);
                const int nw = pos - l + 1;
                double *logit = (double *)malloc(sizeof(double) * (nw + m));
                double *sc = (double *)malloc(sizeof(double) * S);
                double *oc = (double *)malloc(sizeof(double) * (size_t)(m > 0 ? m : 1) * d);
                for (int j = 0; j < nw; ++j) logit[j] = tau * dot(qi, kb + (size_t)(l + j) * d, d);
                for (int u = 0; u < m; ++u) {
                    const int c = sel[u];
                    logit[nw + u] = retrieval_score(p, qhi, k_sum, b_sum, b, h, c);
                    for (int j = 0; j < S; ++j) sc[j] = tau * dot(qi, kb + (size_t)(c * S + j) * d, d);
                    const double Lc = logsumexp(sc, S);
                    for (int t = 0; t < d; ++t) oc[(size_t)u * d + t] = 0.0;
                    for (int j = 0; j < S; ++j) {
                        const double pij = exp(sc[j] - Lc);
                        for (int t = 0; t < d; ++t) oc[(size_t)u * d + t] += pij * vb[(size_t)(c * S + j) * d + t];
                    }
                }
                const double logZ = logsumexp(logit, nw + m);
                double *o = out + (((size_t)b * p->Hq + h) * p->T + i) * d;
                for (int t = 0; t < d; ++t) o[t] = 0.0;
                for (int j = 0; j < nw; ++j) {
                    const double a = exp(logit[j] - logZ);
                    for (int t = 0; t < d; ++t) o[t] += a * vb[(size_t)(l + j) * d + t];
                }
                for (int u = 0; u < m; ++u) {
                    const double beta = exp(logit[nw + u] - logZ);
                    for (int t = 0; t < d; ++t) o[t] += beta * oc[(size_t)u * d + t];
                }
                lse[((size_t)b * p->Hq + h) * p->T + i] = logZ;
                free(sel);
                free(logit);
                free(sc);
                free(oc);
            }
}

/*
 * Eq. 10 evaluated token by token, written independently of orc_attn_fwd so the two can be
 * compared: for every attended token j the explicit weight
 *   w_ij = exp(s_ij) / Z_{i,c(j)} * Z^_{i,c(j)} / Z^_i,
 * with Z_{i,c} = sum_{j in c} exp(s_ij), Z^_{i,c} = exp(s^_{i,c}) for a selected chunk, and for
 * the window segment Z^_{i,win} = Z_{i,win} (its exact mass), Z^_i = Z_{i,win} + sum_sel exp(s^).
 * Returns out = sum_j w_ij v_j and wsum = sum_j w_ij. No max-subtraction: callers keep logits small.
 */
void orc_eq10_tokenwise(const orc_params *p, const double *q, const double *k, const double *v,
                        const double *q_hat, const double *k_sum, const double *b_sum, const int *idx,
                        double *out, double *wsum) {
    const int d = p->d, S = p->S, G = p->Hq / p->Hkv, K = p->topk;
    const double tau = tau_of(p);
    for (int b = 0; b < p->B; ++b)
        for (int h = 0; h < p->Hq; ++h)
            for (int i = 0; i < p->T; ++i) {
                const int g = h / G, pos = p->q_pos0 + i;
                const int l = window_left(p, pos), n = l / S;
                const double *qi = q + (((size_t)b * p->Hq + h) * p->T + i) * d;
                const double *qhi = q_hat + (((size_t)b * p->Hq + h) * p->T + i) * d;
                const double *kb = k + ((size_t)b * p->Hkv + g) * (size_t)p->L * d;
                const double *vb = v + ((size_t)b * p->Hkv + g) * (size_t)p->L * d;
                int *sel = (int *)malloc(sizeof(int) * (K > 0 ? K : 1));
                const int m = selected_set(idx + (((size_t)b * p->Hkv + g) * p->T + i) * K, K, n, sel);
                double Zwin = 0.0;
                for (int j = l; j <= pos; ++j) Zwin += exp(tau * dot(qi, kb + (size_t)j * d, d));
                double Zhat = Zwin;
                for (int u = 0; u < m; ++u) Zhat += exp(retrieval_score(p, qhi, k_sum, b_sum, b, h, sel[u]));
                double *o = out + (((size_t)b * p->Hq + h) * p->T + i) * d;
                for (int t = 0; t < d; ++t) o[t] = 0.0;
                double ws = 0.0;
                for (int j = l; j <= pos; ++j) {
                    const double w = exp(tau * dot(qi, kb + (size_t)j * d, d)) / Zwin * (Zwin / Zhat);
                    ws += w;
                    for (int t = 0; t < d; ++t) o[t] += w * vb[(size_t)j * d + t];
                }
                for (int u = 0; u < m; ++u) {
                    const int c = sel[u];
                    double Zc = 0.0;
                    for (int j = c * S; j < (c + 1) * S; ++j) Zc += exp(tau * dot(qi, kb + (size_t)j * d, d));
                    const double Zhc = exp(retrieval_score(p, qhi, k_sum, b_sum, b, h, c));
                    for (int j = c * S; j < (c + 1) * S; ++j) {
                        const double w = exp(tau * dot(qi, kb + (size_t)j * d, d)) / Zc * (Zhc / Zhat);
                        ws += w;
                        for (int t = 0; t < d; ++t) o[t] += w * vb[(size_t)j * d + t];
                    }
                }
                wsum[((size_t)b * p->Hq + h) * p->T + i] = ws;
                free(sel);
            }
}

/*
 * Gradients of L = sum(dout * out) for the forward above, with the selection idx held fixed
 * (the hard top-k is not differentiable; Sec. 3 RQ2: gradients reach the landmark summaries
 * through s^ in Z^). Notation per (b, h, i): alpha_j = exp(s_j - lse) on the window,
 * beta_c = exp(s^_c - lse), pi_cj = exp(s_j - L_c), D = dout . out.
 *   window: ds_j = alpha_j (dout.v_j - D),  dv_j += alpha_j dout
 *   chunk : ds^_c = beta_c (dout.o_c - D),  ds_j = beta_c pi_cj (dout.v_j - dout.o_c),
 *           dv_j += beta_c pi_cj dout
 *   dq += tau ds_j k_j, dk_j += tau ds_j q, dq^ += tau ds^_c k'_c, dk'_c += tau ds^_c q^, db'_c += ds^_c
 *   Eq. 8 backward per (b, h, c): du_j = p_j (dk'.(k_j - k') - db' (log p_j + b')),
 *           dq'_c = tau sum_j du_j k_j,  dk_j += p_j dk' + tau du_j q'_c.
 * dk/dv accumulate over the G heads of a KV group. Outputs are fully overwritten.
 * Pinned by: central finite differences of orc_chunk_summary + orc_attn_fwd in fp64.
 */
void orc_attn_bwd(const orc_params *p, const double *q, const double *k, const double *v, const double *q_hat,
                  const double *q_land, const int *idx, const double *dout, double *dq, double *dk, double *dv,
                  double *dq_hat, double *dq_land) {
    const int d = p->d, S = p->S, G = p->Hq / p->Hkv, K = p->topk, Nc = p->L / p->S;
    const double tau = tau_of(p);
    const size_t nsum = (size_t)p->B * p->Hq * Nc;
    double *k_sum = (double *)calloc(nsum * d + 1, sizeof(double));
    double *b_sum = (double *)calloc(nsum + 1, sizeof(double));
    double *dk_sum = (double *)calloc(nsum * d + 1, sizeof(double));
    double *db_sum = (double *)calloc(nsum + 1, sizeof(double));
    double *o_fwd = (double *)calloc((size_t)p->B * p->Hq * p->T * d + 1, sizeof(double));
    double *lse = (double *)calloc((size_t)p->B * p->Hq * p->T + 1, sizeof(double));
    orc_chunk_summary(p, k, q_land, 0, Nc, k_sum, b_sum);
    orc_attn_fwd(p, q, k, v, q_hat, k_sum, b_sum, idx, o_fwd, lse);
    memset(dq, 0, sizeof(double) * (size_t)p->B * p->Hq * p->T * d);
    memset(dq_hat, 0, sizeof(double) * (size_t)p->B * p->Hq * p->T * d);
    memset(dk, 0, sizeof(double) * (size_t)p->B * p->Hkv * p->L * d);
    memset(dv, 0, sizeof(double) * (size_t)p->B * p->Hkv * p->L * d);
    memset(dq_land, 0, sizeof(double) * nsum * d);

    /* One (b, KV group) owns its dk, dv, dk', db' slices, so groups run in parallel. */
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < p->B; ++b)
        for (int g = 0; g < p->Hkv; ++g) {
            const double *kb = k + ((size_t)b * p->Hkv + g) * (size_t)p->L * d;
            const double *vb = v + ((size_t)b * p->Hkv + g) * (size_t)p->L * d;
            double *dkb = dk + ((size_t)b * p->Hkv + g) * (size_t)p->L * d;
            double *dvb = dv + ((size_t)b * p->Hkv + g) * (size_t)p->L * d;
            double *sc = (double *)malloc(sizeof(double) * S);
            double *oc = (double *)malloc(sizeof(double) * d);
            for (int hh = 0; hh < G; ++hh) {
                const int h = g * G + hh;
                for (int i = 0; i < p->T; ++i) {
                    const int pos = p->q_pos0 + i;
                    const int l = window_left(p, pos), n = l / S;
                    const size_t row = ((size_t)b * p->Hq + h) * p->T + i;
                    const double *qi = q + row * d, *qhi = q_hat + row * d, *doi = dout + row * d;
                    const double lz = lse[row];
                    const double D = dot(doi, o_fwd + row * d, d);
                    double *dqi = dq + row * d, *dqhi = dq_hat + row * d;
                    for (int j = l; j <= pos; ++j) {
                        const double s = tau * dot(qi, kb + (size_t)j * d, d);
                        const double a = exp(s - lz);
                        const double ds = a * (dot(doi, vb + (size_t)j * d, d) - D);
                        for (int t = 0; t < d; ++t) {
                            dqi[t] += tau * ds * kb[(size_t)j * d + t];
                            dkb[(size_t)j * d + t] += tau * ds * qi[t];
                            dvb[(size_t)j * d + t] += a * doi[t];
                        }
                    }
                    int *sel = (int *)malloc(sizeof(int) * (K > 0 ? K : 1));
                    const int m = selected_set(idx + (((size_t)b * p->Hkv + g) * p->T + i) * K, K, n, sel);
                    for (int u = 0; u < m; ++u) {
                        const int c = sel[u];
                        const size_t crow = ((size_t)b * p->Hq + h) * Nc + c;
                        const double shat = tau * dot(qhi, k_sum + crow * d, d) + b_sum[crow];
                        const double beta = exp(shat - lz);
                        for (int j = 0; j < S; ++j) sc[j] = tau * dot(qi, kb + (size_t)(c * S + j) * d, d);
                        const double Lc = logsumexp(sc, S);
                        for (int t = 0; t < d; ++t) oc[t] = 0.0;
                        for (int j = 0; j < S; ++j) {
                            const double pij = exp(sc[j] - Lc);
                            for (int t = 0; t < d; ++t) oc[t] += pij * vb[(size_t)(c * S + j) * d + t];
                        }
                        const double doo = dot(doi, oc, d);
                        const double dshat = beta * (doo - D);
                        for (int t = 0; t < d; ++t) {
                            dqhi[t] += tau * dshat * k_sum[crow * d + t];
                            dk_sum[crow * d + t] += tau * dshat * qhi[t];
                        }
                        db_sum[crow] += dshat;
                        for (int j = 0; j < S; ++j) {
                            const size_t tok = (size_t)(c * S + j);
                            const double pij = exp(sc[j] - Lc);
                            const double ds = beta * pij * (dot(doi, vb + tok * d, d) - doo);
                            for (int t = 0; t < d; ++t) {
                                dqi[t] += tau * ds * kb[tok * d + t];
                                dkb[tok * d + t] += tau * ds * qi[t];
                                dvb[tok * d + t] += beta * pij * doi[t];
                            }
                        }
                    }
                    free(sel);
                }
                /* Eq. 8 backward for every chunk of this head. */
                for (int c = 0; c < Nc; ++c) {
                    const size_t crow = ((size_t)b * p->Hq + h) * Nc + c;
                    const double *ql = q_land + crow * d;
                    const double *ks = k_sum + crow * d;
                    const double *dks = dk_sum + crow * d;
                    const double dbs = db_sum[crow];
                    for (int j = 0; j < S; ++j) sc[j] = tau * dot(ql, kb + (size_t)(c * S + j) * d, d);
                    const double lu = logsumexp(sc, S);
                    const double dks_ks = dot(dks, ks, d);
                    double *dql = dq_land + crow * d;
                    for (int j = 0; j < S; ++j) {
                        const size_t tok = (size_t)(c * S + j);
                        const double logp = sc[j] - lu;
                        const double pj = exp(logp);
                        const double du = pj * (dot(dks, kb + tok * d, d) - dks_ks - dbs * (logp + b_sum[crow]));
                        for (int t = 0; t < d; ++t) {
                            dql[t] += tau * du * kb[tok * d + t];
                            dkb[tok * d + t] += pj * dks[t] + tau * du * ql[t];
                        }
                    }
                }
            }
            free(sc);
            free(oc);
        }
    free(k_sum);
    free(b_sum);
    free(dk_sum);
    free(db_sum);
    free(o_fwd);
    free(lse);
}
