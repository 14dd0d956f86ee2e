/*
 * hsa_oracle.c -- plain, slow, CPU reference for Hierarchical Sparse Attention (HSA).
 *
 * TEST INFRASTRUCTURE ONLY. This file is the oracle that the CUDA path is checked against.
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg may load it; the
 * product path never calls it and shares no code with it.
 *
 * Source: "Every Token Counts: Generalizing 16M Ultra-Long Context in Large Language Models",
 * explainer page (agent-atlas), section "How It Works (Technically)":
 *   Step 1  chunks of S = 64 tokens, one landmark per chunk;
 *   Step 2  retrieval score s[t,i] = Q[t].L[i] / sqrt(d) over the chunks that come before t,
 *           and the top-K set I_t;
 *   Step 3  attention inside each selected chunk separately, one output per chunk;
 *   Step 4  fusion weights w = softmax of the selected retrieval scores, O_t = sum_i w_i O[t,i].
 * and section "The algorithm, simplified" (the per-token procedure: score every past chunk,
 * stable sort by score descending and keep the first top_k, attend each, softmax-weighted sum).
 *
 * Readings of points the page leaves open (each is stated again where it is used):
 *   R1 causal rule: chunk c is admissible for token t iff the chunk has ended at or before t,
 *      i.e. chunk*(c+1) - 1 <= t, so the number of admissible chunks is n_t = (t+1) / chunk.
 *   R2 a token with no admissible chunk gets O = 0, no selection (index -1, weight 0).
 *   R3 n_t < K: every admissible chunk is selected and the fusion softmax runs over those only.
 *   R4 ties: the stable descending sort keeps equal scores in ascending chunk order, so the
 *      lower chunk index wins.
 *   R5 one scale for both retrieval and in-chunk logits (the caller passes it, normally 1/sqrt(D)).
 *   R6 one query serves as both the retrieval query and the attention query unless a separate
 *      retrieval query Qs is passed; no positional encoding.
 *   R7 query-key normalisation (Step 3, norm(.)) is an option (qk_norm): when on, the attention
 *      query and every key are replaced by x / max(||x||_2, 1e-6) before their dot product; the
 *      retrieval scores (Step 2) and the values are left as given. When off, inputs are used as given.
 *   R8 grouped heads: H query heads share Hkv key/value/landmark heads (H a multiple of Hkv);
 *      query head h reads head h / (H / Hkv) of K, V and L. Every query head scores and selects
 *      on its own. Hkv == H is the plain one-to-one case.
 *
 * Arithmetic: inputs arrive as float arrays holding bf16-exact values; every product and sum is
 * accumulated in double. Parallelism is over independent rows only (OpenMP when compiled with
 * -fopenmp), so the result does not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_ENOMEM (-2)

/* R1: number of chunks that have ended at or before position t. */
static int64_t admissible_chunks(int64_t t, int64_t chunk) { return (t + 1) / chunk; }

#define QK_NORM_EPS 1e-6

/*
 * R7: the vector that Step 3 uses for x (a query or a key), in double: norm(x) = x / max(||x||_2, eps)
 * with query-key normalisation, x itself without.
 */
static void attn_vector(const float *x, int64_t D, int qk_norm, double *y) {
    double n = 1.0;
    if (qk_norm) {
        double n2 = 0.0;
        for (int64_t d = 0; d < D; ++d) n2 += (double)x[d] * (double)x[d];
        n = fmax(sqrt(n2), QK_NORM_EPS);
    }
    for (int64_t d = 0; d < D; ++d) y[d] = (double)x[d] / n;
}

/*
 * Gradient through y = x / max(||x||, eps). On entry g = dLoss/dy, on return dLoss/dx:
 * (g - y (y.g)) / ||x|| when ||x|| > eps (the derivative of x / ||x||), g / eps otherwise (there y is
 * x scaled by the constant 1/eps).
 */
static void l2norm_backward(const float *x, int64_t D, double *g) {
    double n2 = 0.0;
    for (int64_t d = 0; d < D; ++d) n2 += (double)x[d] * (double)x[d];
    const double n = sqrt(n2);
    if (n > QK_NORM_EPS) {
        double yg = 0.0;
        for (int64_t d = 0; d < D; ++d) yg += (double)x[d] / n * g[d];
        for (int64_t d = 0; d < D; ++d) g[d] = (g[d] - (double)x[d] / n * yg) / n;
    } else {
        for (int64_t d = 0; d < D; ++d) g[d] /= QK_NORM_EPS;
    }
}

/* Step 2 score for one (query, landmark) pair: scale * sum_d q[d] * l[d], in double. */
static double retrieval_score(const float *q, const float *l, int64_t D, double scale) {
    double acc = 0.0;
    for (int64_t d = 0; d < D; ++d) acc += (double)q[d] * (double)l[d];
    return scale * acc;
}

/*
 * Stable sort of idx[0..n) by score descending (bottom-up merge sort; on equal scores the element
 * that came first stays first). This is the "sorted(range(n), key=score, reverse=True)" of the
 * page's per-token procedure; with idx initialised to 0..n-1, equal scores end in ascending index
 * order (R4).
 */
static void stable_sort_desc(const double *score, int64_t *idx, int64_t *tmp, int64_t n) {
    for (int64_t width = 1; width < n; width *= 2) {
        for (int64_t lo = 0; lo < n; lo += 2 * width) {
            int64_t mid = lo + width < n ? lo + width : n;
            int64_t hi = lo + 2 * width < n ? lo + 2 * width : n;
            int64_t a = lo, b = mid, o = lo;
            while (a < mid && b < hi) {
                /* take from the right run only when strictly greater: keeps stability */
                if (score[idx[b]] > score[idx[a]]) tmp[o++] = idx[b++];
                else tmp[o++] = idx[a++];
            }
            while (a < mid) tmp[o++] = idx[a++];
            while (b < hi) tmp[o++] = idx[b++];
        }
        memcpy(idx, tmp, (size_t)n * sizeof(int64_t));
    }
}

/*
 * Step 2 top-K: fills sel[0..k) with the first k = min(topk, n) entries of the stable descending
 * order of score[0..n), sel_s with their scores, and *next with the score of entry k (the best
 * unselected chunk), or -INFINITY when every chunk was selected. Returns k, or -1 on no memory.
 */
static int64_t select_topk(const double *score, int64_t n, int64_t topk, int64_t *sel, double *sel_s,
                           double *next) {
    int64_t k = n < topk ? n : topk;
    *next = -INFINITY;
    if (n == 0) return 0;
    int64_t *idx = (int64_t *)malloc((size_t)n * sizeof(int64_t));
    int64_t *tmp = (int64_t *)malloc((size_t)n * sizeof(int64_t));
    if (!idx || !tmp) { free(idx); free(tmp); return -1; }
    for (int64_t c = 0; c < n; ++c) idx[c] = c;
    stable_sort_desc(score, idx, tmp, n);
    for (int64_t j = 0; j < k; ++j) { sel[j] = idx[j]; sel_s[j] = score[idx[j]]; }
    if (k < n) *next = score[idx[k]];
    free(idx);
    free(tmp);
    return k;
}

/*
 * Step 3: ordinary softmax attention of one query against one chunk's keys and values.
 * qa is the query as Step 3 uses it (attn_vector); each key likewise goes through attn_vector (R7).
 * logits a_u = scale * qa.ka_u; P = softmax(a) (max-subtracted, the usual stable form of the same
 * function); o = sum_u P_u V[u]. Kc and Vc are [chunk, D] row-major; p receives P (length chunk).
 */
static void attend_one_chunk(const double *qa, const float *Kc, const float *Vc, int64_t chunk, int64_t D,
                             double scale, int qk_norm, double *o, double *p) {
    double m = -INFINITY;
    double ka[D];
    for (int64_t u = 0; u < chunk; ++u) {
        attn_vector(Kc + u * D, D, qk_norm, ka);
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) acc += qa[d] * ka[d];
        p[u] = scale * acc;
        if (p[u] > m) m = p[u];
    }
    double z = 0.0;
    for (int64_t u = 0; u < chunk; ++u) { p[u] = exp(p[u] - m); z += p[u]; }
    for (int64_t u = 0; u < chunk; ++u) p[u] /= z;
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t u = 0; u < chunk; ++u)
        for (int64_t d = 0; d < D; ++d) o[d] += p[u] * (double)Vc[u * D + d];
}

/* Step 4 weights: w_j = exp(s_j - max s) / sum_i exp(s_i - max s) over the k selected scores. */
static void fusion_weights(const double *sel_s, int64_t k, double *w) {
    if (k == 0) return;
    double m = sel_s[0];
    for (int64_t j = 1; j < k; ++j) if (sel_s[j] > m) m = sel_s[j];
    double z = 0.0;
    for (int64_t j = 0; j < k; ++j) { w[j] = exp(sel_s[j] - m); z += w[j]; }
    for (int64_t j = 0; j < k; ++j) w[j] /= z;
}

/*
 * Steps 3 and 4 for one token given its selected chunks: chunk_k[j] / chunk_v[j] point at the
 * [chunk, D] keys / values of the j-th selected chunk, sel_s[j] is its retrieval score.
 * out[D] = sum_j w_j * attend(q, chunk j); w[0..k) receives the weights.
 */
static int attend_and_fuse(const float *q, const float *const *chunk_k, const float *const *chunk_v,
                           const double *sel_s, int64_t k, int64_t chunk, int64_t D, double scale, int qk_norm,
                           double *out, double *w) {
    for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
    if (k == 0) return ORACLE_OK; /* R2 */
    double *o = (double *)malloc((size_t)D * sizeof(double));
    double *p = (double *)malloc((size_t)chunk * sizeof(double));
    double *qa = (double *)malloc((size_t)D * sizeof(double));
    if (!o || !p || !qa) { free(o); free(p); free(qa); return ORACLE_ENOMEM; }
    fusion_weights(sel_s, k, w);
    attn_vector(q, D, qk_norm, qa);
    for (int64_t j = 0; j < k; ++j) {
        attend_one_chunk(qa, chunk_k[j], chunk_v[j], chunk, D, scale, qk_norm, o, p);
        for (int64_t d = 0; d < D; ++d) out[d] += w[j] * o[d];
    }
    free(o);
    free(p);
    free(qa);
    return ORACLE_OK;
}

/*
 * HSA forward for a list of rows.
 *   Q : [B, H, T, D]   K, V : [B, Hkv, T, D]   L : [B, Hkv, N, D] with N = T / chunk (one landmark
 *   per complete chunk); query head h uses key/value/landmark head h / (H / Hkv) (R8)
 *   Qs      : [B, H, T, D] separate retrieval queries, or NULL (Q retrieves too)
 *   qk_norm : query-key normalisation in Step 3 (R7), 0 or 1
 *   rows    : nrows flat row ids r = (b*H + h)*T + t, or NULL for all B*H*T rows in order
 * Outputs, per listed row i (row-major in i):
 *   out[i, D]; sel_idx[i, topk] (chunk ids in the stable descending order, -1 padding);
 *   sel_w[i, topk] (fusion weights, 0 padding); sel_s[i, topk] (scores, 0 padding);
 *   next_s[i] = score of the best unselected admissible chunk, -INFINITY if none.
 * Any output pointer except out may be NULL.
 */
int hsa_oracle_forward_rows(const float *Q, const float *Qs, const float *K, const float *V, const float *L, int64_t B,
                            int64_t H, int64_t Hkv, int64_t T, int64_t D, int64_t chunk, int64_t topk, double scale,
                            int qk_norm, int64_t nrows, const int64_t *rows, double *out, int32_t *sel_idx,
                            double *sel_w, double *sel_s, double *next_s) {
    if (!Q || !K || !V || !L || !out || B < 0 || H < 0 || T < 0 || D < 1 || chunk < 1 || topk < 1 || Hkv < 1 ||
        H % Hkv != 0)
        return ORACLE_EINVAL;
    const int64_t G = H / Hkv;
    const int64_t N = T / chunk;
    if (!rows) nrows = B * H * T;
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 16) reduction(min : status)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t r = rows ? rows[i] : i;
        if (r < 0 || r >= B * H * T) { status = ORACLE_EINVAL; continue; }
        int64_t bh = r / T, t = r % T;
        int64_t kvh = (bh / H) * Hkv + (bh % H) / G;  /* R8: the key/value/landmark head */
        const float *q = Q + r * D;
        const float *qs = (Qs ? Qs : Q) + r * D;  /* retrieval query (Step 2); q attends (Step 3) */
        int64_t n = admissible_chunks(t, chunk);
        if (n > N) n = N;
        double *score = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
        int64_t *sel = (int64_t *)malloc((size_t)topk * sizeof(int64_t));
        double *ss = (double *)calloc((size_t)topk, sizeof(double));
        double *w = (double *)calloc((size_t)topk, sizeof(double));
        const float **ck = (const float **)malloc((size_t)topk * sizeof(float *));
        const float **cv = (const float **)malloc((size_t)topk * sizeof(float *));
        if (!score || !sel || !ss || !w || !ck || !cv) {
            status = ORACLE_ENOMEM;
        } else {
            for (int64_t c = 0; c < n; ++c) score[c] = retrieval_score(qs, L + (kvh * N + c) * D, D, scale);
            double nxt;
            int64_t k = select_topk(score, n, topk, sel, ss, &nxt);
            if (k < 0) {
                status = ORACLE_ENOMEM;
            } else {
                for (int64_t j = 0; j < k; ++j) {
                    ck[j] = K + (kvh * T + sel[j] * chunk) * D;
                    cv[j] = V + (kvh * T + sel[j] * chunk) * D;
                }
                if (attend_and_fuse(q, ck, cv, ss, k, chunk, D, scale, qk_norm, out + i * D, w) != ORACLE_OK)
                    status = ORACLE_ENOMEM;
                for (int64_t j = 0; j < topk; ++j) {
                    if (sel_idx) sel_idx[i * topk + j] = j < k ? (int32_t)sel[j] : -1;
                    if (sel_w) sel_w[i * topk + j] = j < k ? w[j] : 0.0;
                    if (sel_s) sel_s[i * topk + j] = j < k ? ss[j] : 0.0;
                }
                if (next_s) next_s[i] = nxt;
            }
        }
        free(score); free(sel); free(ss); free(w); free(ck); free(cv);
    }
    return status;
}

/*
 * All admissible retrieval scores of a list of rows (used to judge near-ties).
 * Q : [B, H, T, D] (the retrieval queries), L : [B, Hkv, N, D] (R8).
 * scores[i, 0..N) = s[t, c] for c < n_t, and NaN for chunks that are not admissible.
 */
int hsa_oracle_scores_rows(const float *Q, const float *L, int64_t B, int64_t H, int64_t Hkv, int64_t T, int64_t D,
                           int64_t chunk, double scale, int64_t nrows, const int64_t *rows, double *scores) {
    if (!Q || !L || !rows || !scores || D < 1 || chunk < 1 || Hkv < 1 || H % Hkv != 0) return ORACLE_EINVAL;
    const int64_t N = T / chunk, G = H / Hkv;
    int status = ORACLE_OK;
#pragma omp parallel for schedule(static) reduction(min : status)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t r = rows[i];
        if (r < 0 || r >= B * H * T) { status = ORACLE_EINVAL; continue; }
        int64_t bh = r / T, t = r % T;
        int64_t kvh = (bh / H) * Hkv + (bh % H) / G;
        int64_t n = admissible_chunks(t, chunk);
        if (n > N) n = N;
        for (int64_t c = 0; c < N; ++c)
            scores[i * N + c] = c < n ? retrieval_score(Q + r * D, L + (kvh * N + c) * D, D, scale) : NAN;
    }
    return status;
}

/*
 * Decode retrieval (Step 2 for one new token per sequence against a cached history).
 *   q : [B, H, D] (the retrieval queries)   Lc : [B, Hkv, Nmax, D] (R8)   cache_len[b] : tokens in
 *   sequence b's cache
 * The new token sees every chunk that is complete in its cache: n = cache_len / chunk (R1 with
 * the query placed at the last cached position). Outputs per (b, h): sel_idx, sel_s, sel_w
 * [B, H, topk] as in hsa_oracle_forward_rows, and next_s [B, H]. all_s (optional, [B, H, Nmax]) receives
 * every retrieval score of Step 2, NaN for the chunks the token does not see: what a near-tie judgement
 * of another selection needs.
 */
int hsa_oracle_decode_select(const float *q, const float *Lc, const int64_t *cache_len, int64_t B, int64_t H,
                             int64_t Hkv, int64_t D, int64_t Nmax, int64_t chunk, int64_t topk, double scale,
                             int32_t *sel_idx, double *sel_s, double *sel_w, double *next_s, double *all_s) {
    if (!q || !Lc || !cache_len || !sel_idx || D < 1 || chunk < 1 || topk < 1 || Hkv < 1 || H % Hkv != 0)
        return ORACLE_EINVAL;
    const int64_t G = H / Hkv;
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : status)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        int64_t b = bh / H;
        int64_t kvh = b * Hkv + (bh % H) / G;
        int64_t n = cache_len[b] / chunk;
        if (n > Nmax) n = Nmax;
        if (n < 0) n = 0;
        double *score = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
        int64_t *sel = (int64_t *)malloc((size_t)topk * sizeof(int64_t));
        double *ss = (double *)calloc((size_t)topk, sizeof(double));
        double *w = (double *)calloc((size_t)topk, sizeof(double));
        if (!score || !sel || !ss || !w) {
            status = ORACLE_ENOMEM;
        } else {
            for (int64_t c = 0; c < n; ++c) score[c] = retrieval_score(q + bh * D, Lc + (kvh * Nmax + c) * D, D, scale);
            if (all_s)
                for (int64_t c = 0; c < Nmax; ++c) all_s[bh * Nmax + c] = c < n ? score[c] : NAN;
            double nxt;
            int64_t k = select_topk(score, n, topk, sel, ss, &nxt);
            if (k < 0) {
                status = ORACLE_ENOMEM;
            } else {
                fusion_weights(ss, k, w);
                for (int64_t j = 0; j < topk; ++j) {
                    sel_idx[bh * topk + j] = j < k ? (int32_t)sel[j] : -1;
                    if (sel_s) sel_s[bh * topk + j] = j < k ? ss[j] : 0.0;
                    if (sel_w) sel_w[bh * topk + j] = j < k ? w[j] : 0.0;
                }
                if (next_s) next_s[bh] = nxt;
            }
        }
        free(score); free(sel); free(ss); free(w);
    }
    return status;
}

/*
 * Steps 3 and 4 for R independent tokens whose selected chunks are given gathered:
 *   q  : [R, D]            Lg : [R, topk, D]          (landmarks of the selected chunks)
 *   Kg, Vg : [R, topk, chunk, D]                      (keys / values of the selected chunks)
 *   nsel[i] : how many of the topk slots of row i are selected (the first nsel[i])
 *   qs : [R, D] separate retrieval queries or NULL;  qk_norm : R7 in Step 3
 * out[R, D], sel_w[R, topk] (0 padding). The retrieval scores are recomputed from qs (else q) and Lg.
 * Used for decode (with chunks gathered from a cache too large for host memory) and to evaluate
 * the HSA output of a given selection.
 */
int hsa_oracle_attend_gathered(const float *q, const float *qs, const float *Lg, const float *Kg, const float *Vg,
                               const int32_t *nsel, int64_t R, int64_t D, int64_t chunk, int64_t topk,
                               double scale, int qk_norm, double *out, double *sel_w) {
    if (!q || !Lg || !Kg || !Vg || !nsel || !out || D < 1 || chunk < 1 || topk < 1) return ORACLE_EINVAL;
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 4) reduction(min : status)
    for (int64_t i = 0; i < R; ++i) {
        int64_t k = nsel[i];
        if (k < 0 || k > topk) { status = ORACLE_EINVAL; continue; }
        double *ss = (double *)calloc((size_t)topk, sizeof(double));
        double *w = (double *)calloc((size_t)topk, sizeof(double));
        const float **ck = (const float **)malloc((size_t)topk * sizeof(float *));
        const float **cv = (const float **)malloc((size_t)topk * sizeof(float *));
        if (!ss || !w || !ck || !cv) {
            status = ORACLE_ENOMEM;
        } else {
            for (int64_t j = 0; j < k; ++j) {
                ss[j] = retrieval_score((qs ? qs : q) + i * D, Lg + (i * topk + j) * D, D, scale);
                ck[j] = Kg + (i * topk + j) * chunk * D;
                cv[j] = Vg + (i * topk + j) * chunk * D;
            }
            if (attend_and_fuse(q + i * D, ck, cv, ss, k, chunk, D, scale, qk_norm, out + i * D, w) != ORACLE_OK)
                status = ORACLE_ENOMEM;
            if (sel_w)
                for (int64_t j = 0; j < topk; ++j) sel_w[i * topk + j] = j < k ? w[j] : 0.0;
        }
        free(ss); free(w); free(ck); free(cv);
    }
    return status;
}

/*
 * Backward of the HSA forward for a FIXED selection (the top-K choice is a discrete step with no
 * gradient; the gradient reaches the landmarks only through the selected scores, which is how the
 * explainer's Step 4 says retrieval is learned: w multiplies the output, so dLoss/ds flows).
 *
 *   Q, dO : [B, H, T, D]   K, V : [B, Hkv, T, D]   L : [B, Hkv, N, D] (R8)
 *   sel_idx : [B, H, T, topk] (-1 = empty slot)
 *   Qs : [B, H, T, D] retrieval queries, or NULL when Q also retrieves (then dQs must be NULL too)
 *   qk_norm : R7 in Step 3
 * Outputs (overwritten): dQ [B, H, T, D], dK, dV [B, Hkv, T, D], dL [B, Hkv, N, D], all double; with a
 * separate Qs, dQ holds the attention part only and dQs [B, H, T, D] the retrieval part (the ds L terms).
 *
 * Chain rule, per row t with selected chunks j (scores s_j, weights w = softmax(s)); qa and ka_u are
 * the query and keys as Step 3 uses them (attn_vector: normalised under R7, else as given):
 *   O_j  = P_j V_j,  P_j = softmax(a_j),  a_j[u] = scale * qa.ka_u        (Step 3)
 *   O    = sum_j w_j O_j                                                  (Step 4)
 *   dO_j = w_j dO;   dw_j = dO.O_j;   ds_j = w_j (dw_j - sum_i w_i dw_i)  (softmax Jacobian)
 *   dV_j[u] += P_j[u] dO_j;   dP_j[u] = dO_j.V_j[u];
 *   da_j[u] = P_j[u] (dP_j[u] - sum_v P_j[v] dP_j[v])
 *   dqa += scale sum_u da_j[u] ka_u;   dka_u += scale da_j[u] qa;
 *   dq_retrieval += scale ds_j L_j;    dL_j += scale ds_j q_retrieval.
 * Then dq = dqa and dk = dka without R7; with R7 both go back through the normalisation
 * (l2norm_backward). The key/value/landmark gradients of one head collect every query head of its
 * group; the group's query heads, and the rows inside each, are processed in order and the
 * (b, key head) slices in parallel, so the accumulation order is fixed.
 */
int hsa_oracle_backward(const float *Q, const float *Qs, const float *K, const float *V, const float *L,
                        const float *dO, const int32_t *sel_idx, int64_t B, int64_t H, int64_t Hkv, int64_t T,
                        int64_t D, int64_t chunk, int64_t topk, double scale, int qk_norm, double *dQ, double *dK,
                        double *dV, double *dL, double *dQs) {
    if (!Q || !K || !V || !L || !dO || !sel_idx || !dQ || !dK || !dV || !dL || D < 1 || chunk < 1 || topk < 1 ||
        Hkv < 1 || H % Hkv != 0)
        return ORACLE_EINVAL;
    if ((Qs == NULL) != (dQs == NULL)) return ORACLE_EINVAL;
    const int64_t N = T / chunk, G = H / Hkv;
    memset(dQ, 0, (size_t)(B * H * T * D) * sizeof(double));
    if (dQs) memset(dQs, 0, (size_t)(B * H * T * D) * sizeof(double));
    memset(dK, 0, (size_t)(B * Hkv * T * D) * sizeof(double));
    memset(dV, 0, (size_t)(B * Hkv * T * D) * sizeof(double));
    memset(dL, 0, (size_t)(B * Hkv * N * D) * sizeof(double));
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : status)
    for (int64_t kvh = 0; kvh < B * Hkv; ++kvh) {
        double *s = (double *)malloc((size_t)topk * sizeof(double));
        double *w = (double *)malloc((size_t)topk * sizeof(double));
        double *dw = (double *)malloc((size_t)topk * sizeof(double));
        double *Oj = (double *)malloc((size_t)(topk * D) * sizeof(double));
        double *Pj = (double *)malloc((size_t)(topk * chunk) * sizeof(double));
        int64_t *cj = (int64_t *)malloc((size_t)topk * sizeof(int64_t));
        double *dP = (double *)malloc((size_t)chunk * sizeof(double));
        double *qa = (double *)malloc((size_t)D * sizeof(double));
        double *ka = (double *)malloc((size_t)D * sizeof(double));
        double *dqa = (double *)malloc((size_t)D * sizeof(double));
        if (!s || !w || !dw || !Oj || !Pj || !cj || !dP || !qa || !ka || !dqa) {
            status = ORACLE_ENOMEM;
        } else {
            const int64_t b = kvh / Hkv, hk = kvh % Hkv;
            for (int64_t g = 0; g < G; ++g) {
                const int64_t bh = b * H + hk * G + g;  /* R8: the query heads of this key head */
                for (int64_t t = 0; t < T; ++t) {
                    const int64_t r = bh * T + t;
                    const float *q = Q + r * D;
                    const float *qs = (Qs ? Qs : Q) + r * D;  /* retrieval query */
                    double *dq_ret = (dQs ? dQs : dQ) + r * D;  /* its gradient */
                    const float *go = dO + r * D;
                    int64_t k = 0;
                    for (int64_t j = 0; j < topk; ++j) {
                        int32_t c = sel_idx[r * topk + j];
                        if (c < 0) continue;
                        if (c >= N || c >= admissible_chunks(t, chunk)) { status = ORACLE_EINVAL; continue; }
                        cj[k++] = c;
                    }
                    if (k == 0) continue;
                    attn_vector(q, D, qk_norm, qa);
                    for (int64_t d = 0; d < D; ++d) dqa[d] = 0.0;
                    for (int64_t j = 0; j < k; ++j) s[j] = retrieval_score(qs, L + (kvh * N + cj[j]) * D, D, scale);
                    fusion_weights(s, k, w);
                    double wdw = 0.0;
                    for (int64_t j = 0; j < k; ++j) {
                        const float *Kc = K + (kvh * T + cj[j] * chunk) * D;
                        const float *Vc = V + (kvh * T + cj[j] * chunk) * D;
                        attend_one_chunk(qa, Kc, Vc, chunk, D, scale, qk_norm, Oj + j * D, Pj + j * chunk);
                        double acc = 0.0;
                        for (int64_t d = 0; d < D; ++d) acc += (double)go[d] * Oj[j * D + d];
                        dw[j] = acc;
                        wdw += w[j] * acc;
                    }
                    for (int64_t j = 0; j < k; ++j) {
                        const int64_t c = cj[j];
                        const float *Kc = K + (kvh * T + c * chunk) * D;
                        const float *Vc = V + (kvh * T + c * chunk) * D;
                        const float *Lc = L + (kvh * N + c) * D;
                        double *dKc = dK + (kvh * T + c * chunk) * D;
                        double *dVc = dV + (kvh * T + c * chunk) * D;
                        double *dLc = dL + (kvh * N + c) * D;
                        const double *P = Pj + j * chunk;
                        const double ds = w[j] * (dw[j] - wdw);
                        double pdp = 0.0;
                        for (int64_t u = 0; u < chunk; ++u) {
                            double acc = 0.0;
                            for (int64_t d = 0; d < D; ++d) acc += (double)go[d] * (double)Vc[u * D + d];
                            dP[u] = w[j] * acc;
                            pdp += P[u] * dP[u];
                        }
                        for (int64_t u = 0; u < chunk; ++u) {
                            const double da = P[u] * (dP[u] - pdp);
                            attn_vector(Kc + u * D, D, qk_norm, ka);
                            for (int64_t d = 0; d < D; ++d) {
                                dVc[u * D + d] += P[u] * w[j] * (double)go[d];
                                dqa[d] += scale * da * ka[d];
                                dKc[u * D + d] += scale * da * qa[d];  /* dLoss/dka while R7 is on */
                            }
                        }
                        for (int64_t d = 0; d < D; ++d) {
                            dq_ret[d] += scale * ds * (double)Lc[d];
                            dLc[d] += scale * ds * (double)qs[d];
                        }
                    }
                    if (qk_norm) l2norm_backward(q, D, dqa);
                    for (int64_t d = 0; d < D; ++d) dQ[r * D + d] += dqa[d];
                }
            }
            if (qk_norm)  /* every key of this head: dLoss/dka back through the normalisation */
                for (int64_t u = 0; u < T; ++u) l2norm_backward(K + (kvh * T + u) * D, D, dK + (kvh * T + u) * D);
        }
        free(s); free(w); free(dw); free(Oj); free(Pj); free(cj); free(dP); free(qa); free(ka); free(dqa);
    }
    return status;
}
