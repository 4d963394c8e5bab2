/*
 * lsa_oracle.c -- CPU oracle for the Lookahead Sparse Attention (LSA) decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path (the
 * CUDA library and its Python binding) never calls, links or imports it, and it
 * shares no code, header, table or helper with that path.
 *
 * Plain, slow, single-threaded, obviously-correct definitions.  All floating
 * point work is done in fp64; bf16 inputs are widened exactly (a bf16 value is
 * the top 16 bits of an IEEE fp32 value).  fp32 score arrays given as inputs are
 * used exactly as given.
 *
 * Sources (arXiv 2606.09079, "FlashMemory-DeepSeek-V4: Lightning Index
 * Ultra-Long Context via Lookahead Sparse Attention", as described on):
 *   [gist 2.1]  gist.science explainer, "Technisches Resuemee", section 2.1
 *               (periodic trigger tau=64, lookahead index score I_{t,s},
 *               sigmoid gating, fetch of every entry with I >= 0.5, staged
 *               Lightning-Indexer top-k inside the fetched set)
 *   [gist 2.4]  same page, section 2.4 (three independent indexers at layers
 *               10, 12 and 20, their predictions combined by a union, OR mode)
 *   [gist 2.2]  same page, section 2.2 (softmax -> top-p 0.6 -> at least
 *               theta = 3 layers vote)
 *   [cjcn 2]    cjcn.com.cn article, section 2 (trigger every 64 steps, ReLU
 *               replaced by Sigmoid, threshold 0.5, second-stage top-k, the
 *               most recent 8000 tokens always resident on the GPU)
 *   [cjcn 4]    same article, section 4 (one independent memory indexer at
 *               each of layers 10, 12 and 20; a chunk is recalled when any of
 *               the three scores it at 0.5 or more: "OR-mode routing")
 *   [gist 2.3]  same page, section 2.3 (frozen compressed keys; only the
 *               low-rank projection matrices of the query encoder are trained)
 *   [cjcn 5]    same article, section 5 (results: the baselines are a pure
 *               sliding window keeping the recent 8K, and random retention of
 *               10 % of the history chunks; all schemes keep the recent window)
 *   [gist 4]    same page, section 4 ("Recency Only" and "Random 10%" baselines)
 *   [cjcn 3]    same article, section 3 (cross-layer majority vote labelling:
 *               softmax, nucleus top-p 0.6, selected by at least 3 layers,
 *               golden blocks of all steps in the window merged)
 *
 * Readings taken where the pages are silent (each one is listed in the design
 * notes with its reason):
 *   - the score I_{t,s} is sigma(sum_h w_h * (q_h . K_s)): per-head dot products,
 *     a weighted head sum, one sigmoid; no 1/sqrt(d) scale;
 *   - a chunk is kept iff I >= 0.5;
 *   - the Lightning-Indexer score of token t is sum_h w_h * ReLU(q_h . k_t) over
 *     tokens of kept chunks that lie before the recent window;
 *   - top-k keeps the k largest scores, ties to the lower token position, and
 *     reports the kept positions in ascending order;
 *   - attention is softmax(scale * q_h . K_j) over S = top-k rows plus the
 *     window [window_start, window_start + window_len); for the latent (MLA)
 *     layout V_j is the first dv columns of the K row;
 *   - nucleus: the smallest prefix of the descending order whose cumulative
 *     probability reaches top_p, the crossing element included; ties in the
 *     order go to the lower chunk index;
 *   - vote mode 0: a chunk is positive if at some step at least min_layers
 *     layers select it at that same step; mode 1: at least min_layers distinct
 *     layers select it at any steps of the window.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define LSAO_CHUNK 64 /* tokens per KV chunk */

enum { LSAO_OK = 0, LSAO_ERR_ARG = 1, LSAO_ERR_CAPACITY = 4, LSAO_ERR_TABLE = 6 };

static double bf16_value(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------- */
/* a1: Neural Memory Indexer chunk score and 0.5 gate  [gist 2.1] [cjcn 2]    */
/* ------------------------------------------------------------------------- */

/* Logit of one chunk: per-head dot products, then the weighted head sum. */
static double nmi_logit(const uint16_t *q, const uint16_t *w, const uint16_t *khat_row, int Hn, int dn)
{
    double total = 0.0;
    for (int h = 0; h < Hn; ++h) {
        double dot = 0.0;
        for (int d = 0; d < dn; ++d)
            dot += bf16_value(q[(size_t)h * dn + d]) * bf16_value(khat_row[d]);
        total += bf16_value(w[h]) * dot;
    }
    return total;
}

/*
 * For every sequence b and every chunk s of it: I = sigmoid(logit); keep iff
 * I >= 0.5.  Kept chunk indices (relative to the sequence) are written in
 * ascending order.  Returns LSAO_ERR_CAPACITY if a sequence keeps more than
 * kept_cap chunks (its list is then truncated to kept_cap entries and
 * kept_count holds the untruncated count).
 *   q [B, Hn, dn] bf16, w [B, Hn] bf16, khat [total_chunks, dn] bf16,
 *   seq_chunk_offset [B+1], kept_idx [B, kept_cap] (unused slots = -1),
 *   kept_count [B], logits/probs [total_chunks] (optional).
 */
int lsao_nmi_select(const uint16_t *q, const uint16_t *w, const uint16_t *khat,
                    const int64_t *seq_chunk_offset, int B, int Hn, int dn,
                    int32_t *kept_idx, int32_t *kept_count, int kept_cap,
                    double *logits, double *probs)
{
    int status = LSAO_OK;
    if (B < 0 || Hn <= 0 || dn <= 0 || kept_cap < 0)
        return LSAO_ERR_ARG;
    for (int b = 0; b < B; ++b) {
        int64_t first = seq_chunk_offset[b];
        int64_t n_ch = seq_chunk_offset[b + 1] - first;
        int count = 0;
        for (int j = 0; j < kept_cap; ++j)
            kept_idx[(size_t)b * kept_cap + j] = -1;
        for (int64_t s = 0; s < n_ch; ++s) {
            double logit = nmi_logit(q + (size_t)b * Hn * dn, w + (size_t)b * Hn,
                                     khat + (size_t)(first + s) * dn, Hn, dn);
            double prob = 1.0 / (1.0 + exp(-logit));
            if (logits) logits[first + s] = logit;
            if (probs) probs[first + s] = prob;
            if (prob >= 0.5) {
                if (count < kept_cap)
                    kept_idx[(size_t)b * kept_cap + count] = (int32_t)s;
                else
                    status = LSAO_ERR_CAPACITY;
                ++count;
            }
        }
        kept_count[b] = count;
    }
    return status;
}

/*
 * OR-mode routing over several independent indexers  [cjcn 4] [gist 2.4]:
 * the deployed configuration places one indexer at each of three layers; each
 * has its own queries, head weights and compressed keys and scores every chunk
 * exactly as lsao_nmi_select does, and a chunk is fetched when ANY of them
 * gives it a score of at least 0.5.  Kept chunk indices are written in
 * ascending order; capacity is handled as in lsao_nmi_select.
 *   q[i] [B, Hn, dn], w[i] [B, Hn], khat[i] [total_chunks, dn] for indexer i.
 */
int lsao_nmi_select_union(int n_idx, const uint16_t *const *q, const uint16_t *const *w,
                          const uint16_t *const *khat, const int64_t *seq_chunk_offset, int B,
                          int Hn, int dn, int32_t *kept_idx, int32_t *kept_count, int kept_cap)
{
    int status = LSAO_OK;
    if (n_idx <= 0 || B < 0 || Hn <= 0 || dn <= 0 || kept_cap < 0)
        return LSAO_ERR_ARG;
    for (int b = 0; b < B; ++b) {
        int64_t first = seq_chunk_offset[b];
        int64_t n_ch = seq_chunk_offset[b + 1] - first;
        int count = 0;
        for (int j = 0; j < kept_cap; ++j)
            kept_idx[(size_t)b * kept_cap + j] = -1;
        for (int64_t s = 0; s < n_ch; ++s) {
            int fetched = 0;
            for (int i = 0; i < n_idx; ++i) {
                double logit = nmi_logit(q[i] + (size_t)b * Hn * dn, w[i] + (size_t)b * Hn,
                                         khat[i] + (size_t)(first + s) * dn, Hn, dn);
                double prob = 1.0 / (1.0 + exp(-logit));
                if (prob >= 0.5)
                    fetched = 1;
            }
            if (fetched > 0) {
                if (count < kept_cap)
                    kept_idx[(size_t)b * kept_cap + count] = (int32_t)s;
                else
                    status = LSAO_ERR_CAPACITY;
                ++count;
            }
        }
        kept_count[b] = count;
    }
    return status;
}

/* ------------------------------------------------------------------------- */
/* a2: Lightning-Indexer token score  [gist 2.1 "Gestufte Selektion"] [cjcn 2] */
/* ------------------------------------------------------------------------- */

/* score(t) = sum_h w_h * max(0, q_h . k_t) for each of n key rows. */
int lsao_li_scores(const uint16_t *q_li, const uint16_t *w_li, const uint16_t *keys,
                   int n, int Hl, int dl, double *out)
{
    if (n < 0 || Hl <= 0 || dl <= 0)
        return LSAO_ERR_ARG;
    for (int t = 0; t < n; ++t) {
        double total = 0.0;
        for (int h = 0; h < Hl; ++h) {
            double dot = 0.0;
            for (int d = 0; d < dl; ++d)
                dot += bf16_value(q_li[(size_t)h * dl + d]) * bf16_value(keys[(size_t)t * dl + d]);
            if (dot < 0.0) dot = 0.0;
            total += bf16_value(w_li[h]) * dot;
        }
        out[t] = total;
    }
    return LSAO_OK;
}

/* ------------------------------------------------------------------------- */
/* a3: top-k by full sort  (ties -> lower index; output ascending)            */
/* ------------------------------------------------------------------------- */

struct keyed { double key; int32_t idx; };

static int by_key_desc_then_idx(const void *a, const void *b)
{
    const struct keyed *x = (const struct keyed *)a, *y = (const struct keyed *)b;
    if (x->key > y->key) return -1;
    if (x->key < y->key) return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

static int by_int_asc(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Selects min(k, n) indices of the largest scores; writes them ascending. */
int lsao_topk_select(const double *scores, int n, int k, int32_t *out, int32_t *out_count)
{
    if (n < 0 || k < 0)
        return LSAO_ERR_ARG;
    struct keyed *all = (struct keyed *)malloc(sizeof(struct keyed) * (size_t)(n > 0 ? n : 1));
    if (!all) return LSAO_ERR_ARG;
    for (int i = 0; i < n; ++i) { all[i].key = scores[i]; all[i].idx = i; }
    qsort(all, (size_t)n, sizeof(struct keyed), by_key_desc_then_idx);
    int m = k < n ? k : n;
    for (int i = 0; i < m; ++i) out[i] = all[i].idx;
    qsort(out, (size_t)m, sizeof(int32_t), by_int_asc);
    *out_count = m;
    free(all);
    return LSAO_OK;
}

/* Same selection on fp32 keys taken exactly as given. */
int lsao_topk_select_f32(const float *scores, int n, int k, int32_t *out, int32_t *out_count)
{
    if (n < 0 || k < 0)
        return LSAO_ERR_ARG;
    double *wide = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    if (!wide) return LSAO_ERR_ARG;
    for (int i = 0; i < n; ++i) wide[i] = (double)scores[i];   /* exact widening */
    int rc = lsao_topk_select(wide, n, k, out, out_count);
    free(wide);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* Memory-indexer query encoder  [gist 2.1, 2.3] [cjcn 4]                     */
/* ------------------------------------------------------------------------- */

/*
 * The indexer maps the hidden state h_t of the current token to low-rank
 * indexer queries; only these low-rank projections are trained, and their rank
 * is 2048 in the pages' configuration.  Reading taken (the pages give no
 * formula): a down-projection to the rank, then an up-projection to the heads,
 * and the per-head weights projected from h_t directly, with no normalisation
 * or nonlinearity in between:
 *   c = W_down h           (rank entries)
 *   q = W_up c             (Hn * dn entries, head-major: q[h][d] = entry h * dn + d)
 *   w = W_head h           (Hn entries)
 * for each of the B tokens.  Weights are [out, in] row-major, inputs bf16.
 */
int lsao_query_encoder(const uint16_t *h, int B, int d_model, const uint16_t *w_down, int rank,
                       const uint16_t *w_up, const uint16_t *w_head, int Hn, int dn,
                       double *q_out, double *w_out)
{
    if (B < 0 || d_model <= 0 || rank <= 0 || Hn <= 0 || dn <= 0)
        return LSAO_ERR_ARG;
    double *c = (double *)malloc(sizeof(double) * (size_t)rank);
    if (!c) return LSAO_ERR_ARG;
    for (int b = 0; b < B; ++b) {
        const uint16_t *hb = h + (size_t)b * d_model;
        for (int i = 0; i < rank; ++i) {
            double acc = 0.0;
            for (int k = 0; k < d_model; ++k)
                acc += bf16_value(w_down[(size_t)i * d_model + k]) * bf16_value(hb[k]);
            c[i] = acc;
        }
        for (int o = 0; o < Hn * dn; ++o) {
            double acc = 0.0;
            for (int i = 0; i < rank; ++i)
                acc += bf16_value(w_up[(size_t)o * rank + i]) * c[i];
            q_out[(size_t)b * Hn * dn + o] = acc;
        }
        for (int o = 0; o < Hn; ++o) {
            double acc = 0.0;
            for (int k = 0; k < d_model; ++k)
                acc += bf16_value(w_head[(size_t)o * d_model + k]) * bf16_value(hb[k]);
            w_out[(size_t)b * Hn + o] = acc;
        }
    }
    free(c);
    return LSAO_OK;
}

/* ------------------------------------------------------------------------- */
/* Baseline selectors  [cjcn 5] [gist 4]                                      */
/* ------------------------------------------------------------------------- */

/*
 * Output number c (counting from 0) of a SplitMix64 stream started at `seed`
 * (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
 * OOPSLA 2014): the state advances by the golden-ratio increment before each
 * output, and each output is the state passed through the generator's mixing
 * function.
 */
static uint64_t splitmix64_output(uint64_t seed, uint64_t c)
{
    uint64_t z = seed + (c + 1) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/*
 * The two baselines the pages compare LSA with.  Every scheme keeps the recent
 * window; they differ only in the older history, the n_old = window_start / 64
 * chunks before it.
 *   mode 0, recency only: no older chunk is kept.
 *   mode 1, random fraction: exactly m = floor((n_old * keep_num + keep_den / 2)
 *     / keep_den) older chunks are kept (keep_num / keep_den = 1 / 10 for the
 *     pages' "random 10 %"), chosen uniformly at random: chunk s of sequence b
 *     draws u = (output number b * 2^32 + s of SplitMix64(seed)) >> 40, and the
 *     m chunks with the smallest draws are kept, ties to the lower index.
 * Kept lists are ascending; capacity as in lsao_nmi_select.
 */
int lsao_select_baseline(int mode, const int32_t *window_start, int B, uint64_t seed, int keep_num,
                         int keep_den, int32_t *kept_idx, int32_t *kept_count, int kept_cap)
{
    if ((mode != 0 && mode != 1) || B < 0 || kept_cap < 0 || keep_num < 0 || keep_den <= 0)
        return LSAO_ERR_ARG;
    int status = LSAO_OK;
    for (int b = 0; b < B; ++b) {
        int32_t *out = kept_idx + (size_t)b * kept_cap;
        for (int j = 0; j < kept_cap; ++j)
            out[j] = -1;
        int n_old = window_start[b] > 0 ? window_start[b] / LSAO_CHUNK : 0;
        int64_t m = mode == 0 ? 0 : ((int64_t)n_old * keep_num + keep_den / 2) / keep_den;
        if (m > n_old) m = n_old;
        if (m == 0) { kept_count[b] = 0; continue; }
        /* smallest draws first = largest negated draws first, ties to the lower index */
        double *neg = (double *)malloc(sizeof(double) * (size_t)n_old);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_old);
        int32_t cnt = 0;
        if (!neg || !sel) { free(neg); free(sel); return LSAO_ERR_ARG; }
        for (int c = 0; c < n_old; ++c) {
            uint64_t u = splitmix64_output(seed, ((uint64_t)b << 32) + (uint64_t)c) >> 40;
            neg[c] = -(double)u;
        }
        lsao_topk_select(neg, n_old, (int)m, sel, &cnt);
        for (int j = 0; j < cnt; ++j) {
            if (j < kept_cap) out[j] = sel[j];
            else status = LSAO_ERR_CAPACITY;
        }
        kept_count[b] = cnt;
        free(neg);
        free(sel);
    }
    return status;
}

/* ------------------------------------------------------------------------- */
/* a4: softmax attention over an explicit row set  [cjcn 2] [gist 2.1]        */
/* ------------------------------------------------------------------------- */

/*
 * Dense two-pass softmax attention of Hq query heads over n rows given by their
 * element offsets into k_base / v_base:
 *   s_hj = scale * q_h . K_j ; o_h = sum_j softmax_j(s_h) V_j ; lse_h = log sum_j exp(s_hj)
 * With n == 0 the output is zero and lse is -inf.
 */
static void attend_rows(const uint16_t *q, int Hq, int dqk, int dv,
                        const uint16_t *k_base, const uint16_t *v_base,
                        const int64_t *k_off, const int64_t *v_off, int n,
                        double scale, double *out, double *lse)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (int h = 0; h < Hq; ++h) {
        const uint16_t *qh = q + (size_t)h * dqk;
        double *oh = out + (size_t)h * dv;
        for (int e = 0; e < dv; ++e) oh[e] = 0.0;
        if (n == 0) { lse[h] = -INFINITY; continue; }
        double mx = -INFINITY;
        for (int j = 0; j < n; ++j) {
            double dot = 0.0;
            for (int d = 0; d < dqk; ++d)
                dot += bf16_value(qh[d]) * bf16_value(k_base[k_off[j] + d]);
            s[j] = scale * dot;
            if (s[j] > mx) mx = s[j];
        }
        double sum = 0.0;
        for (int j = 0; j < n; ++j) {
            double p = exp(s[j] - mx);
            sum += p;
            for (int e = 0; e < dv; ++e)
                oh[e] += p * bf16_value(v_base[v_off[j] + e]);
        }
        for (int e = 0; e < dv; ++e) oh[e] /= sum;
        lse[h] = mx + log(sum);
    }
    free(s);
}

/* Plain attention over n contiguous rows: K [n, k_stride], V [n, v_stride]. */
int lsao_attention_dense(const uint16_t *q, int Hq, int dqk, int dv,
                         const uint16_t *k_rows, int64_t k_stride,
                         const uint16_t *v_rows, int64_t v_stride, int n,
                         double scale, double *out, double *lse)
{
    if (n < 0 || Hq <= 0 || dqk <= 0 || dv <= 0)
        return LSAO_ERR_ARG;
    int64_t *ko = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
    int64_t *vo = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
    for (int j = 0; j < n; ++j) { ko[j] = (int64_t)j * k_stride; vo[j] = (int64_t)j * v_stride; }
    attend_rows(q, Hq, dqk, dv, k_rows, v_rows, ko, vo, n, scale, out, lse);
    free(ko); free(vo);
    return LSAO_OK;
}

/* ------------------------------------------------------------------------- */
/* a2+a3+a4 composed: one decode step of one sequence                         */
/* ------------------------------------------------------------------------- */

/*
 * Token position p lives in row p % 64 of pool slot chunk_table[p / 64].
 * Pools: li_pool [slots, 64, dl]; k_pool [slots, 64, k_row_stride];
 * v_pool [slots, 64, v_row_stride] or NULL for the latent layout, where V is
 * the first dv columns of each k_pool row.
 *
 * Candidates for the fine top-k: every token of every kept chunk whose index is
 * below window_start / 64 (kept chunks inside the window are attended anyway).
 * Candidates are enumerated in ascending kept-chunk order, rows 0..63, i.e. in
 * ascending token position.  S = top-k positions + [window_start, window_start + window_len).
 *
 * Outputs: topk_pos [k] ascending, -1 padded; topk_count; li_scores (optional,
 * one per candidate, in candidate order, n_cand_out receives their number);
 * out [Hq, dv]; lse [Hq].
 */
int lsao_decode_step(const uint16_t *q_li, const uint16_t *w_li, int Hl, int dl,
                     const uint16_t *li_pool,
                     const uint16_t *q, int Hq, int dqk, int dv,
                     const uint16_t *k_pool, int64_t k_row_stride,
                     const uint16_t *v_pool, int64_t v_row_stride, double scale,
                     const int32_t *chunk_table, int n_table,
                     const int32_t *kept_idx, int kept_count,
                     int window_start, int window_len, int k,
                     int32_t *topk_pos, int32_t *topk_count,
                     double *li_scores, int32_t *n_cand_out,
                     double *out, double *lse)
{
    if (window_start < 0 || window_start % LSAO_CHUNK != 0 || window_len < 0 || k < 0 || kept_count < 0)
        return LSAO_ERR_ARG;
    int first_window_chunk = window_start / LSAO_CHUNK;

    /* candidate positions */
    int n_cold = 0;
    for (int j = 0; j < kept_count; ++j)
        if (kept_idx[j] < first_window_chunk) ++n_cold;
    int n_cand = n_cold * LSAO_CHUNK;
    int32_t *cand_pos = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_cand > 0 ? n_cand : 1));
    uint16_t *cand_keys = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(n_cand > 0 ? n_cand : 1) * dl);
    int c = 0;
    for (int j = 0; j < kept_count; ++j) {
        int chunk = kept_idx[j];
        if (chunk >= first_window_chunk) continue;
        if (chunk < 0 || chunk >= n_table || chunk_table[chunk] < 0) {
            free(cand_pos); free(cand_keys);
            return LSAO_ERR_TABLE;
        }
        int64_t slot = chunk_table[chunk];
        for (int r = 0; r < LSAO_CHUNK; ++r, ++c) {
            cand_pos[c] = chunk * LSAO_CHUNK + r;
            memcpy(cand_keys + (size_t)c * dl, li_pool + ((size_t)slot * LSAO_CHUNK + r) * dl,
                   sizeof(uint16_t) * (size_t)dl);
        }
    }

    /* fine scores and top-k */
    double *sc = (double *)malloc(sizeof(double) * (size_t)(n_cand > 0 ? n_cand : 1));
    lsao_li_scores(q_li, w_li, cand_keys, n_cand, Hl, dl, sc);
    if (li_scores) memcpy(li_scores, sc, sizeof(double) * (size_t)n_cand);
    if (n_cand_out) *n_cand_out = n_cand;
    int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)(k > 0 ? k : 1));
    int32_t n_sel = 0;
    lsao_topk_select(sc, n_cand, k, sel, &n_sel);
    for (int i = 0; i < k; ++i) topk_pos[i] = i < n_sel ? cand_pos[sel[i]] : -1;
    *topk_count = n_sel;

    /* attention row set */
    int n_rows = n_sel + window_len;
    int64_t *ko = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_rows > 0 ? n_rows : 1));
    int64_t *vo = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_rows > 0 ? n_rows : 1));
    int status = LSAO_OK;
    for (int j = 0; j < n_rows; ++j) {
        int pos = j < n_sel ? topk_pos[j] : window_start + (j - n_sel);
        int chunk = pos / LSAO_CHUNK;
        if (chunk >= n_table || chunk_table[chunk] < 0) { status = LSAO_ERR_TABLE; break; }
        int64_t row = (int64_t)chunk_table[chunk] * LSAO_CHUNK + pos % LSAO_CHUNK;
        ko[j] = row * k_row_stride;
        vo[j] = row * (v_pool ? v_row_stride : k_row_stride);
    }
    if (status == LSAO_OK)
        attend_rows(q, Hq, dqk, dv, k_pool, v_pool ? v_pool : k_pool, ko, vo, n_rows, scale, out, lse);

    free(cand_pos); free(cand_keys); free(sc); free(sel); free(ko); free(vo);
    return status;
}

/* ------------------------------------------------------------------------- */
/* a7: cross-layer majority-vote labelling  [gist 2.2] [cjcn 3]              */
/* ------------------------------------------------------------------------- */

/*
 * Nucleus of one score vector: softmax (temperature 1), order chunks by score
 * descending (ties -> lower index), keep the smallest prefix whose cumulative
 * probability reaches top_p (the crossing element included; all chunks if the
 * sum never reaches it).  sel[c] = 1 for kept chunks.  Returns the prefix size.
 */
int lsao_nucleus(const float *scores, int n, double top_p, uint8_t *sel)
{
    if (n <= 0) return 0;
    double mx = -INFINITY;
    for (int i = 0; i < n; ++i) if ((double)scores[i] > mx) mx = (double)scores[i];
    struct keyed *ord = (struct keyed *)malloc(sizeof(struct keyed) * (size_t)n);
    double z = 0.0;
    for (int i = 0; i < n; ++i) {
        ord[i].key = (double)scores[i];
        ord[i].idx = i;
        z += exp((double)scores[i] - mx);
    }
    qsort(ord, (size_t)n, sizeof(struct keyed), by_key_desc_then_idx);
    memset(sel, 0, (size_t)n);
    double cum = 0.0;
    int taken = 0;
    for (int i = 0; i < n; ++i) {
        cum += exp(ord[i].key - mx) / z;
        sel[ord[i].idx] = 1;
        ++taken;
        if (cum >= top_p) break;
    }
    free(ord);
    return taken;
}

/*
 * scores [n_layers, n_steps, n_chunks] fp32.  count[t][c] = number of layers
 * whose nucleus at step t contains chunk c.
 *   mode 0: max_votes[c] = max_t count[t][c]; label[c] = max_votes[c] >= min_layers
 *   mode 1: max_votes[c] = number of distinct layers selecting c at any step;
 *           label[c] = max_votes[c] >= min_layers
 */
int lsao_label_vote(const float *scores, int n_layers, int n_steps, int n_chunks,
                    double top_p, int min_layers, int mode,
                    uint8_t *labels, int32_t *max_votes)
{
    if (n_layers <= 0 || n_steps <= 0 || n_chunks <= 0 || (mode != 0 && mode != 1))
        return LSAO_ERR_ARG;
    int32_t *count = (int32_t *)calloc((size_t)n_steps * n_chunks, sizeof(int32_t));
    uint8_t *ever = (uint8_t *)calloc((size_t)n_layers * n_chunks, 1);
    uint8_t *sel = (uint8_t *)malloc((size_t)n_chunks);
    for (int l = 0; l < n_layers; ++l) {
        for (int t = 0; t < n_steps; ++t) {
            const float *row = scores + ((size_t)l * n_steps + t) * n_chunks;
            lsao_nucleus(row, n_chunks, top_p, sel);
            for (int c = 0; c < n_chunks; ++c) {
                if (sel[c]) {
                    count[(size_t)t * n_chunks + c] += 1;
                    ever[(size_t)l * n_chunks + c] = 1;
                }
            }
        }
    }
    for (int c = 0; c < n_chunks; ++c) {
        int best = 0;
        if (mode == 0) {
            for (int t = 0; t < n_steps; ++t)
                if (count[(size_t)t * n_chunks + c] > best) best = count[(size_t)t * n_chunks + c];
        } else {
            for (int l = 0; l < n_layers; ++l) best += ever[(size_t)l * n_chunks + c];
        }
        if (max_votes) max_votes[c] = best;
        labels[c] = (uint8_t)(best >= min_layers);
    }
    free(count); free(ever); free(sel);
    return LSAO_OK;
}
