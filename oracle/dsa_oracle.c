/*
 * dsa_oracle.c -- plain, slow, single-threaded CPU oracle for the DeepSeek
 * Sparse Attention (DSA) layer stack under IndexCache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only the tests, the package's smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header, table or helper with the CUDA
 * library.  All arithmetic is in IEEE double; bf16 inputs arrive as their raw
 * 16-bit patterns and are widened exactly.
 *
 * Sources (two web pages; titles as printed, section named per function):
 *   [IC]  "读懂 IndexCache：从 DSA 的选词开销到跨层索引复用" (ulna520 blog)
 *   [IDX] "注意力机制中的 Index：从位置下标到预算检索" (Jerry's Blog)
 *
 * Readings taken where the pages are silent (each one is listed in the design
 * notes): visibility is s < t; ties in the top-k go to the lower position;
 * -0.0 equals +0.0; a row lists its selected positions in ascending order and
 * pads with -1; a query that sees nothing attends to nothing (output 0,
 * log-sum-exp = -inf); the main-attention logits carry a caller scale.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 -> double: a bf16 is the upper half of an IEEE binary32. */
static double bf(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Lightning indexer score, one query row.
 * [IDX] §4 (DeepSeek-V3.2 token-level lightning indexer), the index-score
 * equation: I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s]).  Candidates are the
 * visible set of [IDX] §1, P_t = {s : 0 <= s < t}.
 *   q_row : [H][d] bf16 bits (the H indexer heads of query t)
 *   k     : [>=T][d] bf16 bits (indexer keys; row s is k[s])
 *   w_row : [H] float (head weights of query t)
 *   T     : number of visible candidates (the query's absolute position)
 *   I_out : [T] scores.  Returns the number of (t,s) pairs scored (= T). */
long long oracle_indexer_row(const uint16_t *q_row, const uint16_t *k,
                             const float *w_row, int H, int d, int T,
                             double *I_out) {
    for (int s = 0; s < T; ++s) {
        double I = 0.0;
        for (int j = 0; j < H; ++j) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c)
                dot += bf(q_row[(size_t)j * d + c]) * bf(k[(size_t)s * d + c]);
            double relu = dot > 0.0 ? dot : 0.0;
            I += (double)w_row[j] * relu;
        }
        I_out[s] = I;
    }
    return (long long)T;
}

/* ------------------------------------------------------------------------ */
/* Top-k selection, one query row.
 * [IDX] §4: S_t = TopK_k { I[t,s] : s < t } and [IC] §1 (k = 2048 in the
 * paper's runs).  Reading: order candidates by (score descending, position
 * ascending), keep the first min(k, T), list them by ascending position and
 * pad with -1 up to k.  Equal scores compare equal even for -0.0 vs +0.0
 * because the comparison is IEEE equality. */
typedef struct { double v; int s; } cand_t;

static int cand_cmp(const void *a, const void *b) {
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->s < y->s) ? -1 : (x->s > y->s);
}

static int int_cmp(const void *a, const void *b) {
    int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/* Returns the number of valid entries written (min(k, T)). */
int oracle_topk_row(const double *I, int T, int k, int32_t *idx_out) {
    cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(T > 0 ? T : 1));
    for (int s = 0; s < T; ++s) { c[s].v = I[s]; c[s].s = s; }
    qsort(c, (size_t)T, sizeof(cand_t), cand_cmp);
    int n = T < k ? T : k;
    int *sel = (int *)malloc(sizeof(int) * (size_t)(n > 0 ? n : 1));
    for (int r = 0; r < n; ++r) sel[r] = c[r].s;
    qsort(sel, (size_t)n, sizeof(int), int_cmp);
    for (int r = 0; r < k; ++r) idx_out[r] = r < n ? sel[r] : -1;
    free(sel);
    free(c);
    return n;
}

/* ------------------------------------------------------------------------ */
/* Shared softmax-attention core over an explicit list of key positions.
 * For each head h: e_r = scale * q[h] . K[pos_r]; alpha = softmax(e);
 * out[h] = sum_r alpha_r V[pos_r][0:Dv].  Empty list -> out = 0, lse = -inf. */
static void attend_list(const uint16_t *q_row, const uint16_t *K, int64_t ks,
                        const uint16_t *V, int64_t vs, const int *pos, int n,
                        int n_h, int Dqk, int Dv, double scale, double *out,
                        double *lse) {
    double *e = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (int h = 0; h < n_h; ++h) {
        double *o = out + (size_t)h * Dv;
        for (int c = 0; c < Dv; ++c) o[c] = 0.0;
        if (n == 0) { if (lse) lse[h] = -INFINITY; continue; }
        double m = -INFINITY;
        for (int r = 0; r < n; ++r) {
            double dot = 0.0;
            const uint16_t *kr = K + (int64_t)pos[r] * ks;
            for (int c = 0; c < Dqk; ++c)
                dot += bf(q_row[(size_t)h * Dqk + c]) * bf(kr[c]);
            e[r] = scale * dot;
            if (e[r] > m) m = e[r];
        }
        double z = 0.0;
        for (int r = 0; r < n; ++r) { e[r] = exp(e[r] - m); z += e[r]; }
        for (int r = 0; r < n; ++r) {
            double a = e[r] / z;
            const uint16_t *vr = V + (int64_t)pos[r] * vs;
            for (int c = 0; c < Dv; ++c) o[c] += a * bf(vr[c]);
        }
        if (lse) lse[h] = m + log(z);
    }
    free(e);
}

/* Sparse core attention, one query row.
 * [IDX] §2, the equations for alpha-hat and o-hat: softmax over exactly the
 * selected set S_t, then the alpha-weighted sum of the selected values; [IDX]
 * §4, u_t = Attn(h_t, {c_s : s in S_t}), where for MLA every query head reads
 * the same latent row (MQA form).  idx holds k entries; -1 entries are padding
 * and are skipped.  Returns the number of valid entries attended. */
int oracle_sparse_attn_row(const uint16_t *q_row, const uint16_t *K, int64_t ks,
                           const uint16_t *V, int64_t vs, const int32_t *idx,
                           int k, int n_h, int Dqk, int Dv, double scale,
                           double *out, double *lse) {
    int *pos = (int *)malloc(sizeof(int) * (size_t)(k > 0 ? k : 1));
    int n = 0;
    for (int r = 0; r < k; ++r)
        if (idx[r] >= 0) pos[n++] = idx[r];
    attend_list(q_row, K, ks, V, vs, pos, n, n_h, Dqk, Dv, scale, out, lse);
    free(pos);
    return n;
}

/* Dense causal attention, one query row: [IDX] §1, e_{t,s} = q_t . k_s over
 * P_t, softmax over P_t, o_t = sum alpha v_s. */
void oracle_dense_attn_row(const uint16_t *q_row, const uint16_t *K, int64_t ks,
                           const uint16_t *V, int64_t vs, int T, int n_h,
                           int Dqk, int Dv, double scale, double *out,
                           double *lse) {
    int *pos = (int *)malloc(sizeof(int) * (size_t)(T > 0 ? T : 1));
    for (int s = 0; s < T; ++s) pos[s] = s;
    attend_list(q_row, K, ks, V, vs, pos, T, n_h, Dqk, Dv, scale, out, lse);
    free(pos);
}

/* Dense attention weights, one query row: [IDX] §8.1 (Captured Attention
 * Mass), the dense weights alpha^dense_{t,s} that the selected set is scored
 * against.  For each head h: e_s = scale * q[h] . K[s] for s in P_t =
 * {0 <= s < T}; alpha[h][s] = exp(e_s - max e) / sum_s' exp(e_s' - max e).
 * Written on its own (not through attend_list) so that its weights and the
 * list form's log-sum-exp are two independent routes.
 *   alpha : [n_h][T] double (written; nothing for T = 0) */
void oracle_dense_probs_row(const uint16_t *q_row, const uint16_t *K, int64_t ks,
                            int T, int n_h, int Dqk, double scale, double *alpha) {
    for (int h = 0; h < n_h; ++h) {
        double *a = alpha + (size_t)h * (size_t)T;
        double m = -INFINITY;
        for (int s = 0; s < T; ++s) {
            double dot = 0.0;
            for (int c = 0; c < Dqk; ++c)
                dot += bf(q_row[(size_t)h * Dqk + c]) * bf(K[(int64_t)s * ks + c]);
            a[s] = scale * dot;
            if (a[s] > m) m = a[s];
        }
        double z = 0.0;
        for (int s = 0; s < T; ++s) { a[s] = exp(a[s] - m); z += a[s]; }
        for (int s = 0; s < T; ++s) a[s] /= z;
    }
}

/* Index-mask formulation, one query row: [IDX] §6.4 (Transformers GLM
 * indexer).  Every position starts at mask -inf, the selected positions are
 * scattered to 0, the causal mask (-inf for s >= t) is added, and a dense
 * softmax runs over all Lk positions.  Written independently of the list
 * form above: it walks every key position and lets exp(-inf) = 0 drop the
 * masked ones. */
void oracle_masked_attn_row(const uint16_t *q_row, const uint16_t *K, int64_t ks,
                            const uint16_t *V, int64_t vs, const int32_t *idx,
                            int k, int T, int Lk, int n_h, int Dqk, int Dv,
                            double scale, double *out, double *lse) {
    double *mask = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
    double *e = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
    for (int s = 0; s < Lk; ++s) mask[s] = -INFINITY;
    for (int r = 0; r < k; ++r)
        if (idx[r] >= 0 && idx[r] < Lk) mask[idx[r]] = 0.0;
    for (int s = 0; s < Lk; ++s)
        if (s >= T) mask[s] += -INFINITY;
    for (int h = 0; h < n_h; ++h) {
        double *o = out + (size_t)h * Dv;
        double m = -INFINITY;
        for (int s = 0; s < Lk; ++s) {
            double dot = 0.0;
            const uint16_t *kr = K + (int64_t)s * ks;
            for (int c = 0; c < Dqk; ++c)
                dot += bf(q_row[(size_t)h * Dqk + c]) * bf(kr[c]);
            e[s] = scale * dot + mask[s];
            if (e[s] > m) m = e[s];
        }
        for (int c = 0; c < Dv; ++c) o[c] = 0.0;
        if (m == -INFINITY) { if (lse) lse[h] = -INFINITY; continue; }
        double z = 0.0;
        for (int s = 0; s < Lk; ++s) { e[s] = exp(e[s] - m); z += e[s]; }
        for (int s = 0; s < Lk; ++s) {
            if (e[s] == 0.0) continue;
            const uint16_t *vr = V + (int64_t)s * vs;
            for (int c = 0; c < Dv; ++c) o[c] += (e[s] / z) * bf(vr[c]);
        }
        if (lse) lse[h] = m + log(z);
    }
    free(e);
    free(mask);
}

/* ------------------------------------------------------------------------ */
/* The IndexCache layer loop over whole (small) inputs.
 * [IC] §1.1 (F layers keep their indexer and select; S layers reuse the most
 * recent F layer's indices; the first layer must be F) and §1.2 with its
 * Figure 2 loop: the cache variable is set on F layers by TopK(indexer(X))
 * and read by every layer's sparse attention; each layer attends with its
 * OWN queries and keys/values.  Projections and the FFN need trained
 * weights; the per-layer tensors are given directly, and no output feeds the
 * next layer.
 *
 * Shapes, per layer l (pointers in arrays of length n_layers):
 *   q_idx[l] [B][Lq][H][dI] bf16, k_idx[l] [B][Lk][dI] bf16, w[l] [B][Lq][H]
 *   (only read on F layers; may be NULL on S layers)
 *   q[l] [B][Lq][n_h][Dqk] bf16, K[l]/V[l] rows of [B][Lk][*] with row
 *   strides ks/vs (elements), out[l] [B][Lq][n_h][Dv] double,
 *   lse[l] [B][Lq][n_h] double (may be NULL).
 *   idx_out[l] [B][Lq][k] int32: the index tensor layer l attended with.
 * Query row i sits at absolute position t = start_pos + i and sees s < t.
 * counters[0] += indexer invocations, counters[1] += scored (t,s) pairs.
 * Returns 0, or -1 if the pattern is invalid (empty, not 'F'/'S', or its
 * first entry is not 'F'). */
int oracle_indexcache_forward(const char *pattern, int n_layers,
                              const uint16_t *const *q_idx,
                              const uint16_t *const *k_idx,
                              const float *const *w, const uint16_t *const *q,
                              const uint16_t *const *K, int64_t ks,
                              const uint16_t *const *V, int64_t vs, int B,
                              int Lq, int Lk, int start_pos, int H, int dI,
                              int k, int n_h, int Dqk, int Dv, double scale,
                              int32_t *const *idx_out, double *const *out,
                              double *const *lse, long long *counters) {
    if (n_layers <= 0 || pattern == NULL || pattern[0] != 'F') return -1;
    for (int l = 0; l < n_layers; ++l)
        if (pattern[l] != 'F' && pattern[l] != 'S') return -1;
    size_t rows = (size_t)B * Lq;
    int32_t *cache = (int32_t *)malloc(sizeof(int32_t) * rows * (size_t)k);
    double *I = (double *)malloc(sizeof(double) * (size_t)(start_pos + Lq + 1));
    for (int l = 0; l < n_layers; ++l) {
        if (pattern[l] == 'F') {
            counters[0] += 1;
            for (int b = 0; b < B; ++b)
                for (int i = 0; i < Lq; ++i) {
                    int T = start_pos + i;
                    size_t row = (size_t)b * Lq + i;
                    counters[1] += oracle_indexer_row(
                        q_idx[l] + row * (size_t)H * dI,
                        k_idx[l] + (size_t)b * Lk * dI, w[l] + row * H, H, dI,
                        T, I);
                    oracle_topk_row(I, T, k, cache + row * k);
                }
        }
        memcpy(idx_out[l], cache, sizeof(int32_t) * rows * (size_t)k);
        for (int b = 0; b < B; ++b)
            for (int i = 0; i < Lq; ++i) {
                size_t row = (size_t)b * Lq + i;
                oracle_sparse_attn_row(
                    q[l] + row * (size_t)n_h * Dqk, K[l] + (int64_t)b * Lk * ks,
                    ks, V[l] + (int64_t)b * Lk * vs, vs, cache + row * k, k,
                    n_h, Dqk, Dv, scale, out[l] + row * (size_t)n_h * Dv,
                    lse && lse[l] ? lse[l] + row * n_h : NULL);
            }
    }
    free(I);
    free(cache);
    return 0;
}
