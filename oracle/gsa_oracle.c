/*
 * GSA oracle — TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU restatement of what the Gist Sparse Attention (GSA)
 * decode path and the gist-causal prefill compute.  Only the tests, the smoke
 * check and the bench's CPU-baseline leg call it; the CUDA library never links
 * or calls it and shares no code with it.
 *
 * Sources (pages about "Forget, Then Recall: Learnable Compression and
 * Selective Unfolding via Gist Sparse Attention", Mao, Li & Fox):
 *   [EN-2]   gist.science explainer (EN), section 2 "Methodology: Gist Sparse
 *            Attention" — interleaved gist tokens, gist as routing signals,
 *            selective unfolding, hybrid attention, hierarchical extension;
 *   [DE-M]   gist.science explainer (DE), section "Methodik";
 *   [EN-4]   gist.science explainer (EN), section 4 "Experimental Results"
 *            (KV-cache reuse: precomputed document caches);
 *   [SL-6]   Taki-lab slide deck (docswell), page 6 "GSA とは" — query scores
 *            every gist, takes top-k, restores the chunks with their gists;
 *   [SL-7]   slide deck, page 7 "Gist token" — gist causal mask example;
 *   [SL-9]   slide deck, page 9 "Training, Stage 1" — the suffix sees gists only;
 *   [SL-10]  slide deck, page 10 "Training, Stage 2" — top-k worked example;
 *   [SL-11]  slide deck, page 11 "Hierarchical Gist-of-Gist Compression";
 *   [SL-17]  slide deck, page 17 "Selective Rules Comparison" — SR-only,
 *            AG+SR, SG+SR;
 *   [SL-18]  slide deck, page 18 "Top-k vs. Top-p";
 *   [DE-E]   gist.science explainer (DE), section "Ergebnisse" (top-p /
 *            nucleus selection).
 *
 * Every floating-point value is widened exactly to double before use; all
 * arithmetic is in double.  Softmax is the two-pass textbook form.
 * Parity status of each function is stated beside it; all are pinned by the
 * CPU tests (worked examples, closed forms, brute force, library routines).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };
enum { OR_ALL_GISTS = 0, OR_SELECTED_PAIRS = 1, OR_SR_ONLY = 2, OR_UNSELECTED_GISTS = 3 };

/* Exact widening of one stored element to double. */
static double ld(const void* p, int dt, int64_t i) {
    if (dt == OR_F64) return ((const double*)p)[i];
    if (dt == OR_F32) return (double)((const float*)p)[i];
    uint32_t u = (uint32_t)((const uint16_t*)p)[i] << 16; /* bf16 bits */
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double default_scale(double scale, int d) { return scale > 0 ? scale : 1.0 / sqrt((double)d); }

/* ------------------------------------------------------------------------ */
/* Step 1 — routing score of every gist.  [EN-2] "Gist as Routing Signals":   */
/* the decoding query is scored against every gist token; [DE-M] "Relevanz-  */
/* Scoring": by dot product with the gist key.  Under grouped-query sharing   */
/* the G query heads of one KV head share one selection, so the score of     */
/* gist j for KV head hk is the sum over the group of the raw logits:        */
/*        s[b,hk,j] = sum_{h in group(hk)} sum_i q[b,h,i] * Kg[b,hk,j,i].    */
/* (No softmax scale: a positive scale does not change the ranking.)         */
/* ------------------------------------------------------------------------ */
/* qb: the query's batch index in q [..][Hq][d] (b for a decode step).      */
static double gist_score_q(int Hq, int Hkv, int d, int N, int dt, const void* q, int64_t qb, const void* kg,
                           int b, int hk, int j) {
    int G = Hq / Hkv;
    double acc = 0.0;
    for (int g = 0; g < G; ++g) {
        int h = hk * G + g;
        for (int i = 0; i < d; ++i)
            acc += ld(q, dt, (qb * Hq + h) * d + i) * ld(kg, dt, (((int64_t)b * Hkv + hk) * N + j) * d + i);
    }
    return acc;
}

static double gist_score(int Hq, int Hkv, int d, int N, int dt, const void* q, const void* kg,
                         int b, int hk, int j) {
    return gist_score_q(Hq, Hkv, d, N, dt, q, b, kg, b, hk, j);
}

void oracle_gist_scores(int B, int Hq, int Hkv, int d, int N, int dt, const void* q, const void* kg,
                        double* s) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < Hkv; ++hk)
            for (int j = 0; j < N; ++j)
                s[((int64_t)b * Hkv + hk) * N + j] = gist_score(Hq, Hkv, d, N, dt, q, kg, b, hk, j);
}

/* ------------------------------------------------------------------------ */
/* Step 2 — top-k chunk selection.  [EN-2] "Selective Unfolding": the k most  */
/* relevant chunks by score; [SL-10] scores 0.1/0.8/0.7/0.2, k=2 -> g2, g3.   */
/* Ties go to the lowest index; the result is listed in ascending order.     */
/* Implementation: sort every (score, index) pair by score descending, index  */
/* ascending; keep the first k; sort those indices ascending.  NaN ranks     */
/* below every number.                                                       */
/* ------------------------------------------------------------------------ */
typedef struct { double s; int32_t j; } scored_t;

static int by_score_desc_then_index(const void* a, const void* b) {
    const scored_t* x = (const scored_t*)a;
    const scored_t* y = (const scored_t*)b;
    int xn = isnan(x->s), yn = isnan(y->s);
    if (xn != yn) return xn ? 1 : -1;
    if (!xn && x->s != y->s) return x->s > y->s ? -1 : 1;
    return (x->j > y->j) - (x->j < y->j);
}

static int by_index(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* Top-k of n scores whose positions are idx_of[0..n) (NULL: 0..n-1). */
static void topk_list(int n, const double* s, const int32_t* idx_of, int k, int32_t* out) {
    scored_t* all = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
    for (int t = 0; t < n; ++t) {
        all[t].s = s[t];
        all[t].j = idx_of ? idx_of[t] : t;
    }
    qsort(all, (size_t)n, sizeof(scored_t), by_score_desc_then_index);
    for (int t = 0; t < k; ++t) out[t] = all[t].j;
    qsort(out, (size_t)k, sizeof(int32_t), by_index);
    free(all);
}

void oracle_topk(int rows, int N, int k, const double* s, int32_t* idx) {
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) topk_list(N, s + (int64_t)r * N, NULL, k, idx + (int64_t)r * k);
}

/* Selection margin of one row: the gap between the k-th and (k+1)-th largest */
/* score (INFINITY when k = 0 or k = n).  Test helper for the decidability     */
/* rule on selected indices.                                                  */
void oracle_topk_gap(int rows, int N, int k, const double* s, double* gap) {
    for (int r = 0; r < rows; ++r) {
        if (k <= 0 || k >= N) { gap[r] = INFINITY; continue; }
        scored_t* all = (scored_t*)malloc(sizeof(scored_t) * (size_t)N);
        for (int t = 0; t < N; ++t) { all[t].s = s[(int64_t)r * N + t]; all[t].j = t; }
        qsort(all, (size_t)N, sizeof(scored_t), by_score_desc_then_index);
        gap[r] = all[k - 1].s - all[k].s;
        free(all);
    }
}

/* ------------------------------------------------------------------------ */
/* Top-p (nucleus) chunk selection.  [SL-18] "Top-k vs. Top-p" and [DE-E]     */
/* "Ergebnisse" compare a fixed top-p selection with top-k; the pages give no */
/* formula.  Reading taken: the routing distribution of a row is the softmax  */
/* of the scaled routing scores, pi_j = exp(scale s_j) / sum_i exp(scale s_i);*/
/* the chunks are taken in the top-k order (higher score first, the lower     */
/* index on ties), and the selection is the shortest prefix of that order     */
/* whose mass reaches p (at least one chunk), cut at kmax.  Output: the       */
/* selected indices ascending, then -1 up to kmax; count[r] = their number.   */
/* ------------------------------------------------------------------------ */
void oracle_topp(int rows, int N, int kmax, double p, double scale, const double* s, int32_t* idx,
                 int32_t* count) {
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        const double* sr = s + (int64_t)r * N;
        scored_t* all = (scored_t*)malloc(sizeof(scored_t) * (size_t)(N > 0 ? N : 1));
        double mx = -INFINITY;
        for (int t = 0; t < N; ++t) {
            all[t].s = sr[t];
            all[t].j = t;
            if (sr[t] > mx) mx = sr[t];
        }
        qsort(all, (size_t)N, sizeof(scored_t), by_score_desc_then_index);
        double z = 0.0;
        for (int t = 0; t < N; ++t) z += exp(scale * (sr[t] - mx));
        int m = 0;
        double acc = 0.0;
        while (m < N && m < kmax) {
            acc += exp(scale * (all[m].s - mx)) / z;
            ++m;
            if (acc >= p) break;
        }
        int32_t* out = idx + (int64_t)r * kmax;
        for (int t = 0; t < m; ++t) out[t] = all[t].j;
        qsort(out, (size_t)m, sizeof(int32_t), by_index);
        for (int t = m; t < kmax; ++t) out[t] = -1;
        count[r] = m;
        free(all);
    }
}

/* Rounding-error bound of an fp32 evaluation of each score, any summation   */
/* order (Higham, "Accuracy and Stability of Numerical Algorithms", 2nd ed., */
/* eq. 3.5, inner products):  |fl(s) - s| <= gamma_n * sum |q_i k_i|,        */
/* gamma_n = n u / (1 - n u), u = 2^-24, n = G*d products summed.  Per row,  */
/* the maximum over the row's gists.                                         */
void oracle_score_error_bound(int B, int Hq, int Hkv, int d, int N, int dt, const void* q,
                              const void* kg, double* eps_row) {
    int G = Hq / Hkv;
    double u = ldexp(1.0, -24), n = (double)G * d;
    double gamma = n * u / (1.0 - n * u);
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < Hkv; ++hk) {
            double worst = 0.0;
            for (int j = 0; j < N; ++j) {
                double acc = 0.0;
                for (int g = 0; g < G; ++g)
                    for (int i = 0; i < d; ++i)
                        acc += fabs(ld(q, dt, ((int64_t)b * Hq + hk * G + g) * d + i) *
                                    ld(kg, dt, (((int64_t)b * Hkv + hk) * N + j) * d + i));
                if (acc > worst) worst = acc;
            }
            eps_row[(int64_t)b * Hkv + hk] = gamma * worst;
        }
}

/* ------------------------------------------------------------------------ */
/* Steps 3-4 — hybrid attention over the assembled context.                  */
/* A context is a list of keys, each a (K row, V row) pair in some tensor.   */
/* For each query head h of the group: l_x = scale * q_h . K_x,              */
/* p_x = exp(l_x - max l) / sum exp(l - max l), out_h = sum_x p_x V_x.       */
/* ------------------------------------------------------------------------ */
typedef struct { const void* k; const void* v; int64_t off; } key_ref;

static void attend(int d, int dt, double scale, const void* q, int64_t q_off, int nkeys,
                   const key_ref* keys, double* out, double* lse) {
    double* logit = (double*)malloc(sizeof(double) * (size_t)(nkeys > 0 ? nkeys : 1));
    double mx = -INFINITY;
    for (int x = 0; x < nkeys; ++x) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += ld(q, dt, q_off + i) * ld(keys[x].k, dt, keys[x].off + i);
        logit[x] = scale * acc;
        if (logit[x] > mx) mx = logit[x];
    }
    double z = 0.0;
    for (int x = 0; x < nkeys; ++x) { logit[x] = exp(logit[x] - mx); z += logit[x]; }
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int x = 0; x < nkeys; ++x) acc += logit[x] * ld(keys[x].v, dt, keys[x].off + i);
        out[i] = nkeys > 0 ? acc / z : NAN;
    }
    if (lse) *lse = nkeys > 0 ? mx + log(z) : NAN;   /* log of sum_x exp(l_x) */
    free(logit);
}

/* Context of one (b, hk) for flat decode.
 * [EN-2] "Hybrid Attention": k raw chunks + their gist tokens + the gist
 * tokens of unselected chunks  -> ALL_GISTS = every gist once, plus the raw
 * tokens of the selected chunks ([SL-17] "AG+SR").
 * [SL-6] / [SL-17] "SG+SR": only the selected chunks' gists and raw tokens
 * -> SELECTED_PAIRS.
 * [SL-17] "SR-only": the selected chunks' raw tokens, no gist at all
 * -> SR_ONLY.
 * [DE-M] "Hybride Attention": the selected raw tokens and the gists of the
 * chunks that were NOT selected (a selected chunk is represented by its raw
 * tokens instead of its gist) -> UNSELECTED_GISTS.
 * In every mode the W uncompressed tail tokens after the last chunk are
 * always attended ([SL-9]: the generation suffix attends directly).          */
/* Element offset of raw token u of chunk j of (b, hk).  Dense: raw [B][Hkv][N][c][d].
 * Paged ([EN-4] "KV-Cache Reuse": precomputed document caches are shared, not
 * copied): chunk j of sequence b is page table[b*N + j] of a pool
 * [pages][Hkv][c][d]; one page holds one chunk of every KV head, so the
 * sequences whose contexts hold the same document point at the same pages. */
static int64_t raw_off(int Hkv, int N, int c, int d, const int32_t* table, int b, int hk, int j, int u) {
    if (table) return (((int64_t)table[(int64_t)b * N + j] * Hkv + hk) * c + u) * d;
    return ((((int64_t)b * Hkv + hk) * N + j) * c + u) * d;
}

/* The context of (b, hk): gists as the mode says (of the sequence's nb <= N
 * chunks), raw tokens of the selected chunks, tail.                         */
static int flat_context(int Hkv, int d, int N, int nb, int c, int W, int mode, int b, int hk, int k,
                        const int32_t* sel, const void* kg, const void* vg, const void* kraw,
                        const void* vraw, const void* ktail, const void* vtail, const int32_t* table,
                        key_ref* keys) {
    int n = 0;
    int64_t row = (int64_t)b * Hkv + hk;
    if (mode == OR_ALL_GISTS) {
        for (int j = 0; j < nb; ++j) keys[n++] = (key_ref){kg, vg, (row * N + j) * d};
    } else if (mode == OR_SELECTED_PAIRS) {
        for (int t = 0; t < k; ++t)
            if (sel[t] >= 0) keys[n++] = (key_ref){kg, vg, (row * N + sel[t]) * d};
    } else if (mode == OR_UNSELECTED_GISTS) {
        for (int j = 0; j < nb; ++j) {
            int selected = 0;
            for (int t = 0; t < k; ++t) selected |= sel[t] == j;
            if (!selected) keys[n++] = (key_ref){kg, vg, (row * N + j) * d};
        }
    }   /* OR_SR_ONLY: no gist */
    for (int t = 0; t < k; ++t)
        if (sel[t] >= 0)   /* -1: an empty place of a variable-size (top-p) selection */
            for (int u = 0; u < c; ++u)
                keys[n++] = (key_ref){kraw, vraw, raw_off(Hkv, N, c, d, table, b, hk, sel[t], u)};
    for (int u = 0; u < W; ++u) keys[n++] = (key_ref){ktail, vtail, (row * W + u) * d};
    return n;
}

/* Full flat decode step: scores (step 1), selection (step 2), hybrid
 * attention (steps 3-4).  Outputs: scores [B*Hkv*N] (may be NULL), selected
 * indices [B*Hkv*k] ascending, out [B*Hq*d].
 * nch (may be NULL: every sequence has N chunks) gives sequence b nb =
 * nch[b] <= N chunks: its gists j >= nb do not exist, so they score -inf,
 * are never selected and are not in the context; with nb < k the selection
 * holds all nb chunks and its other places are empty (-1).                 */
static void decode_impl(int B, int Hq, int Hkv, int d, int N, int c, int k, int W, int mode, double scale,
                        int dt, const void* q, const void* kg, const void* vg, const void* kraw,
                        const void* vraw, const int32_t* table, const int32_t* nch, const void* ktail,
                        const void* vtail, double* scores_out, int32_t* idx_out, double* out) {
    int G = Hq / Hkv;
    double sc = default_scale(scale, d);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < Hkv; ++hk) {
            int64_t row = (int64_t)b * Hkv + hk;
            int nb = nch ? nch[b] : N;
            double* s = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
            for (int j = 0; j < nb; ++j) s[j] = gist_score(Hq, Hkv, d, N, dt, q, kg, b, hk, j);
            if (scores_out)
                for (int j = 0; j < N; ++j) scores_out[row * N + j] = j < nb ? s[j] : -INFINITY;
            int32_t* sel = idx_out + row * k;
            int kk = k < nb ? k : nb;
            topk_list(nb, s, NULL, kk, sel);
            for (int t = kk; t < k; ++t) sel[t] = -1;
            key_ref* keys = (key_ref*)malloc(sizeof(key_ref) * (size_t)(N + (int64_t)k * c + W + 1));
            int nk = flat_context(Hkv, d, N, nb, c, W, mode, b, hk, k, sel, kg, vg, kraw, vraw, ktail,
                                  vtail, table, keys);
            for (int g = 0; g < G; ++g) {
                int h = hk * G + g;
                attend(d, dt, sc, q, ((int64_t)b * Hq + h) * d, nk, keys,
                       out + ((int64_t)b * Hq + h) * d, NULL);
            }
            free(keys);
            free(s);
        }
}

/* Hybrid attention alone, for a given selection idx [B*Hkv*k] (the unfolding
 * + attention step without routing).  lse (may be NULL) [B*Hq] receives the
 * natural log of sum_x exp(scale * q_h . K_x) over the context.              */
static void unfold_impl(int B, int Hq, int Hkv, int d, int N, int c, int k, int W, int mode,
                        double scale, int dt, const void* q, const void* kg, const void* vg,
                        const void* kraw, const void* vraw, const int32_t* table, const void* ktail,
                        const void* vtail, const int32_t* idx, double* out, double* lse) {
    int G = Hq / Hkv;
    double sc = default_scale(scale, d);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < Hkv; ++hk) {
            int64_t row = (int64_t)b * Hkv + hk;
            key_ref* keys = (key_ref*)malloc(sizeof(key_ref) * (size_t)(N + (int64_t)k * c + W + 1));
            int nk = flat_context(Hkv, d, N, N, c, W, mode, b, hk, k, idx + row * k, kg, vg, kraw, vraw,
                                  ktail, vtail, table, keys);
            for (int g = 0; g < G; ++g) {
                int h = hk * G + g;
                attend(d, dt, sc, q, ((int64_t)b * Hq + h) * d, nk, keys,
                       out + ((int64_t)b * Hq + h) * d, lse ? lse + (int64_t)b * Hq + h : NULL);
            }
            free(keys);
        }
}

void oracle_decode(int B, int Hq, int Hkv, int d, int N, int c, int k, int W, int mode, double scale,
                   int dt, const void* q, const void* kg, const void* vg, const void* kraw,
                   const void* vraw, const void* ktail, const void* vtail, double* scores_out,
                   int32_t* idx_out, double* out) {
    decode_impl(B, Hq, Hkv, d, N, c, k, W, mode, scale, dt, q, kg, vg, kraw, vraw, NULL, NULL, ktail, vtail,
                scores_out, idx_out, out);
}

void oracle_unfold_attn(int B, int Hq, int Hkv, int d, int N, int c, int k, int W, int mode,
                        double scale, int dt, const void* q, const void* kg, const void* vg,
                        const void* kraw, const void* vraw, const void* ktail, const void* vtail,
                        const int32_t* idx, double* out, double* lse) {
    unfold_impl(B, Hq, Hkv, d, N, c, k, W, mode, scale, dt, q, kg, vg, kraw, vraw, NULL, ktail, vtail,
                idx, out, lse);
}

/* Decode over a paged raw cache (pools k_pages / v_pages [pages][Hkv][c][d],
 * table [B][N]) with nch[b] chunks in sequence b (nch may be NULL).        */
void oracle_decode_paged(int B, int Hq, int Hkv, int d, int N, int c, int k, int W, int mode, double scale,
                         int dt, const void* q, const void* kg, const void* vg, const void* kpages,
                         const void* vpages, const int32_t* table, const int32_t* nch, const void* ktail,
                         const void* vtail, double* scores_out, int32_t* idx_out, double* out) {
    decode_impl(B, Hq, Hkv, d, N, c, k, W, mode, scale, dt, q, kg, vg, kpages, vpages, table, nch, ktail,
                vtail, scores_out, idx_out, out);
}

/* ------------------------------------------------------------------------ */
/* Hierarchical gist-of-gist decode (H-GSA).  [EN-2] "Hierarchical Extension"*/
/* and [DE-M] "Erweiterung": gists are grouped, a meta-gist summarises each  */
/* group; decoding scores the meta-gists, selects segments, scores the gists */
/* inside the selected segments, then unfolds raw tokens.  [SL-11]: groups  */
/* of consecutive gists (g1..g10 -> G1, ...).                                */
/*   level 2: s2[J] over all n_l2 meta-gists -> S2 = top-k2;                  */
/*   candidates: level-1 gists j with floor(j / group) in S2, ascending;      */
/*   level 1: s1[j] over the candidates -> S1 = top-k1 among them;            */
/*   context: every meta-gist, every candidate gist, raw tokens of S1, tail.  */
/* With given != 0, idx2_out / idx1_out are inputs: the attention is evaluated */
/* for that selection (a test helper for rows whose selection is not decided  */
/* at fp32 precision).                                                        */
/* ------------------------------------------------------------------------ */
void oracle_hier_decode(int B, int Hq, int Hkv, int d, int N1, int c, int k1, int W, int n_l2,
                        int group, int k2, double scale, int dt, const void* q, const void* kg2,
                        const void* vg2, const void* kg1, const void* vg1, const void* kraw,
                        const void* vraw, const void* ktail, const void* vtail, int32_t* idx2_out,
                        int32_t* idx1_out, double* out, int given) {
    int G = Hq / Hkv;
    double sc = default_scale(scale, d);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < Hkv; ++hk) {
            int64_t row = (int64_t)b * Hkv + hk;
            double* s2 = (double*)malloc(sizeof(double) * (size_t)n_l2);
            for (int J = 0; J < n_l2; ++J) s2[J] = gist_score(Hq, Hkv, d, n_l2, dt, q, kg2, b, hk, J);
            int32_t* S2 = idx2_out + row * k2;
            if (!given) topk_list(n_l2, s2, NULL, k2, S2);

            int32_t* cand = (int32_t*)malloc(sizeof(int32_t) * (size_t)k2 * group + 1);
            int nc = 0;
            for (int t = 0; t < k2; ++t)
                for (int u = 0; u < group; ++u) {
                    int j = S2[t] * group + u;
                    if (j < N1) cand[nc++] = j;
                }
            double* s1 = (double*)malloc(sizeof(double) * (size_t)(nc > 0 ? nc : 1));
            for (int t = 0; t < nc; ++t) s1[t] = gist_score(Hq, Hkv, d, N1, dt, q, kg1, b, hk, cand[t]);
            int32_t* S1 = idx1_out + row * k1;
            if (!given) topk_list(nc, s1, cand, k1, S1);

            key_ref* keys = (key_ref*)malloc(sizeof(key_ref) * (size_t)(n_l2 + nc + (int64_t)k1 * c + W + 1));
            int nk = 0;
            for (int J = 0; J < n_l2; ++J) keys[nk++] = (key_ref){kg2, vg2, (row * n_l2 + J) * d};
            for (int t = 0; t < nc; ++t) keys[nk++] = (key_ref){kg1, vg1, (row * N1 + cand[t]) * d};
            for (int t = 0; t < k1; ++t)
                for (int u = 0; u < c; ++u)
                    keys[nk++] = (key_ref){kraw, vraw, ((row * N1 + S1[t]) * c + u) * d};
            for (int u = 0; u < W; ++u) keys[nk++] = (key_ref){ktail, vtail, (row * W + u) * d};
            for (int g = 0; g < G; ++g) {
                int h = hk * G + g;
                attend(d, dt, sc, q, ((int64_t)b * Hq + h) * d, nk, keys,
                       out + ((int64_t)b * Hq + h) * d, NULL);
            }
            free(keys);
            free(s1);
            free(cand);
            free(s2);
        }
}

/* ------------------------------------------------------------------------ */
/* Stage-2 selective finetuning, forward pass.  [EN-2] "Training Procedure": */
/* selective finetuning changes the attention mask so that attention goes    */
/* only to the top-k selected chunks and their raw tokens; [SL-10]: the      */
/* suffix token's attention to the gists gives the scores, the top-k picks   */
/* the chunks to unfold.  Reading taken: every suffix position p selects its */
/* own chunks exactly as a decode query does (the G heads of a KV head share */
/* one selection, summed logits), and attends to the decode context of the   */
/* mode with the suffix tokens 0..p as its tail (causal).                    */
/*   q, out [B][S][Hq][d] (position-major); gists and raw as for decode;     */
/*   ksuf, vsuf [B][Hkv][S][d]; idx_out [B][Hkv][S][k]; scores_out           */
/*   [B][Hkv][S][N] (may be NULL).                                           */
/* ------------------------------------------------------------------------ */
void oracle_suffix_attn(int B, int Hq, int Hkv, int d, int N, int c, int k, int S, int mode, double scale,
                        int dt, const void* q, const void* kg, const void* vg, const void* kraw,
                        const void* vraw, const void* ksuf, const void* vsuf, double* scores_out,
                        int32_t* idx_out, double* out) {
    int G = Hq / Hkv;
    double sc = default_scale(scale, d);
#pragma omp parallel for collapse(3) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < Hkv; ++hk)
            for (int p = 0; p < S; ++p) {
                int64_t row = (int64_t)b * Hkv + hk, qb = (int64_t)b * S + p, yrow = row * S + p;
                double* s = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
                for (int j = 0; j < N; ++j) s[j] = gist_score_q(Hq, Hkv, d, N, dt, q, qb, kg, b, hk, j);
                if (scores_out)
                    for (int j = 0; j < N; ++j) scores_out[yrow * N + j] = s[j];
                int32_t* sel = idx_out + yrow * k;
                topk_list(N, s, NULL, k, sel);
                key_ref* keys = (key_ref*)malloc(sizeof(key_ref) * (size_t)(N + (int64_t)k * c + S + 1));
                int nk = flat_context(Hkv, d, N, N, c, 0, mode, b, hk, k, sel, kg, vg, kraw, vraw, NULL, NULL,
                                      NULL, keys);
                for (int u = 0; u <= p; ++u) keys[nk++] = (key_ref){ksuf, vsuf, (row * S + u) * d};
                for (int g = 0; g < G; ++g) {
                    int h = hk * G + g;
                    attend(d, dt, sc, q, (qb * Hq + h) * d, nk, keys, out + (qb * Hq + h) * d, NULL);
                }
                free(keys);
                free(s);
            }
}

/* ------------------------------------------------------------------------ */
/* Hierarchy of any depth L >= 2 ([EN-2] "Hierarchical Extension (H-GSA)":   */
/* gists are compressed again into higher-level gists and the query descends */
/* coarse to fine; [SL-11] shows the level-2 to level-1 step).  Level 1 has  */
/* one gist per chunk (n[0] = N1); gist J of level l+1 summarises the level-l */
/* gists [J*g, (J+1)*g), g = group[l-1], so n[l] = ceil(n[l-1] / g).  Step:   */
/* every top-level gist is scored and the top k[L-1] taken; at each lower    */
/* level the candidates are the children of the level above's selection (in  */
/* parent order, then child order), scored and cut to the top k[l-1]; the     */
/* raw tokens of the level-1 selection are unfolded.  The context: every     */
/* top-level gist, every candidate of every lower level, the raw tokens of   */
/* the selected chunks, the tail (the two-level step above, one level at a   */
/* time).  kg[l-1], vg[l-1]: the level-l gists [B][Hkv][n[l-1]][d], level 1  */
/* first; idx[l-1] [B][Hkv][k[l-1]] receives level l's selection (given != 0:  */
/* holds it, and the step is evaluated for that selection).                 */
/* ------------------------------------------------------------------------ */
void oracle_hier_levels(int B, int Hq, int Hkv, int d, int c, int W, int L, const int* n, const int* group,
                        const int* k, double scale, int dt, const void* q, const void* const* kg,
                        const void* const* vg, const void* kraw, const void* vraw, const void* ktail,
                        const void* vtail, int32_t* const* idx, double* out, int given) {
    int G = Hq / Hkv;
    double sc = default_scale(scale, d);
    int64_t cap = 0;   /* context keys: bounded by all gists of all levels + raw + tail */
    for (int l = 0; l < L; ++l) cap += n[l];
    cap += (int64_t)k[0] * c + W + 1;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < Hkv; ++hk) {
            int64_t row = (int64_t)b * Hkv + hk;
            key_ref* keys = (key_ref*)malloc(sizeof(key_ref) * (size_t)cap);
            int nk = 0;
            /* top level: every gist is a candidate */
            int top = L - 1;
            int nc = n[top];
            int32_t* cand = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nc > 0 ? nc : 1));
            for (int J = 0; J < nc; ++J) cand[J] = J;
            for (int l = top; l >= 0; --l) {
                /* the candidates of level l+1 (index l) are in the context */
                for (int t = 0; t < nc; ++t) keys[nk++] = (key_ref){kg[l], vg[l], (row * n[l] + cand[t]) * d};
                double* s = (double*)malloc(sizeof(double) * (size_t)(nc > 0 ? nc : 1));
                for (int t = 0; t < nc; ++t) s[t] = gist_score(Hq, Hkv, d, n[l], dt, q, kg[l], b, hk, cand[t]);
                int32_t* S = idx[l] + row * k[l];
                if (!given) topk_list(nc, s, cand, k[l], S);
                free(s);
                if (l == 0) break;
                /* children of the selection, parent by parent */
                int32_t* next = (int32_t*)malloc(sizeof(int32_t) * ((size_t)k[l] * group[l - 1] + 1));
                int m = 0;
                for (int t = 0; t < k[l]; ++t)
                    for (int u = 0; u < group[l - 1]; ++u) {
                        int j = S[t] * group[l - 1] + u;
                        if (j < n[l - 1]) next[m++] = j;
                    }
                free(cand);
                cand = next;
                nc = m;
            }
            for (int t = 0; t < k[0]; ++t)
                for (int u = 0; u < c; ++u)
                    keys[nk++] = (key_ref){kraw, vraw, ((row * n[0] + idx[0][row * k[0] + t]) * c + u) * d};
            for (int u = 0; u < W; ++u) keys[nk++] = (key_ref){ktail, vtail, (row * W + u) * d};
            for (int g = 0; g < G; ++g) {
                int h = hk * G + g;
                attend(d, dt, sc, q, ((int64_t)b * Hq + h) * d, nk, keys, out + ((int64_t)b * Hq + h) * d, NULL);
            }
            free(cand);
            free(keys);
        }
}

/* ------------------------------------------------------------------------ */
/* Gist-causal prefill.  [EN-2] "Interleaved Gist Tokens": the sequence is   */
/* cut into chunks of c tokens and a gist token follows every chunk; a       */
/* gist attends only to its own chunk and to earlier gists.  [SL-7]:         */
/* g1 -> x1,x2; g2 -> g1,x3,x4; g3 -> g1,g2,x5,(x6),g3.  [SL-9]: a token that */
/* follows compressed context sees the gists, not the earlier raw tokens.     */
/* Positions p = 0..N(c+1)-1: chunk(p) = p / (c+1); p is a gist iff          */
/* p mod (c+1) == c.  Query p may attend key t iff t <= p and                */
/*   (t is a gist of an earlier chunk) or (t == p) or                         */
/*   (t is a raw token of p's own chunk).                                    */
/* ------------------------------------------------------------------------ */
int oracle_gist_mask(int64_t p, int64_t t, int c) {
    if (t > p) return 0;
    if (t == p) return 1;
    int64_t cp = p / (c + 1), ct = t / (c + 1);
    int t_gist = (t % (c + 1)) == c;
    if (t_gist) return ct < cp;
    return ct == cp;
}

/* Brute-force count of allowed (query, key) pairs in one sequence. */
int64_t oracle_prefill_pair_count(int N, int c) {
    int64_t P = (int64_t)N * (c + 1), n = 0;
    for (int64_t p = 0; p < P; ++p)
        for (int64_t t = 0; t <= p; ++t) n += oracle_gist_mask(p, t, c);
    return n;
}

/* Prefill output of the listed query rows.  rows: n_rows triples (b, h, p);
 * out: n_rows * d.  q [B][Hq][P][d], k, v [B][Hkv][P][d].                     */
void oracle_prefill_rows(int B, int Hq, int Hkv, int d, int N, int c, double scale, int dt,
                         const void* q, const void* k, const void* v, int64_t n_rows,
                         const int64_t* rows, double* out, double* lse) {
    int G = Hq / Hkv;
    int64_t P = (int64_t)N * (c + 1);
    double sc = default_scale(scale, d);
    (void)B;
#pragma omp parallel for schedule(dynamic)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t b = rows[3 * r], h = rows[3 * r + 1], p = rows[3 * r + 2];
        int64_t hk = h / G;
        key_ref* keys = (key_ref*)malloc(sizeof(key_ref) * (size_t)(p + 1));
        int nk = 0;
        for (int64_t t = 0; t <= p; ++t)
            if (oracle_gist_mask(p, t, c)) keys[nk++] = (key_ref){k, v, ((b * Hkv + hk) * P + t) * d};
        attend(d, dt, sc, q, ((b * Hq + h) * P + p) * d, nk, keys, out + r * d, lse ? lse + r : NULL);
        free(keys);
    }
}
