/*
 * Oracle for exact Top-k sparse decode attention -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct CPU implementation in double precision.
 * It exists to check the CUDA path: only the tests, the package smoke check
 * and the benchmark's CPU-baseline leg may load it.  It shares no code,
 * header or constant with the CUDA library, and the product never calls it.
 *
 * What it computes (per query row r = (b, qpos, h)):
 *   The token variant is exact Top-k decoding as described in "A Preliminary
 *   Study on the Promises and Challenges of Native Top-k Sparse Attention"
 *   (abstract: keep only the keys most similar to the query) and in the
 *   Indexer -> Top-K -> attend workflow of "Sparse Attention in LLM
 *   Inference: Practical Trade-Offs" (section "The Role of the Indexer"),
 *   with the indexer score taken to be the exact scaled dot product:
 *     1. s_i = scale * <q_r, K[b, h / G, i, :]>   for every visible i < vis,
 *        vis = seq_len[b] - Q + qpos + 1 (causal: query qpos of a Q-query
 *        chunk sees the cache up to and including its own position).
 *     2. order the visible positions by (s descending, position ascending)
 *        with a full sort; S = the first min(k, vis) of them (ties at the
 *        k-th score go to the lower position).
 *     3. m = max_i s_i, Z = sum_{i<vis} e^{s_i - m}, Z_k = sum_{i in S} e^{s_i - m}.
 *     4. out = sum_{i in S} (e^{s_i - m} / Z_k) V[b, h / G, i, :]   (softmax over
 *        S only, then P.V over the selected rows).
 *     5. tail = sum_{i not in S} e^{s_i - m} / Z: the discarded softmax tail
 *        mass, which "A Mathematical Theory of Top-k Sparse Attention via
 *        Total Variation Distance" (abstract) identifies with TV(P, P_hat).
 *     6. idx = S in ascending position order, padded with -1 up to k.
 *   The block variant follows the block-sparse / MoBA description of
 *   "Sparse Attention Landscape" (section "Block Sparse Attention"): the
 *   cache of a sequence is cut into blocks of `block_size` tokens, a block's
 *   key is the mean of its keys, a block's score is scale * <q, mean key>,
 *   the top `top_blocks` blocks other than the last one are kept (ties to the
 *   lower block), the last (current) block is always kept, and dense softmax
 *   attention runs over the tokens of the kept blocks.
 *
 * Inputs are either fp32 (dtype 0) or bf16 bit patterns (dtype 1); a bf16
 * value converts to double exactly.  Outputs are double.  Rows are spread over
 * OpenMP threads; each row is computed independently.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_OK = 0, OR_BAD_ARG = 1, OR_NO_MEMORY = 2 };

typedef struct {
    double s;
    int32_t i;
} scored_pos;

static double load_elem(const void *base, int dtype, size_t off) {
    if (dtype == 0) return (double)((const float *)base)[off];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[off]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* (score descending, position ascending) */
static int cmp_score_desc(const void *a, const void *b) {
    const scored_pos *x = (const scored_pos *)a, *y = (const scored_pos *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->i > y->i) - (x->i < y->i);
}

static int cmp_int_asc(const void *a, const void *b) {
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

static double resolve_scale(double scale, int d) { return scale > 0.0 ? scale : 1.0 / sqrt((double)d); }

static int check_shape(int B, int Q, int Hq, int Hkv, int d, int L_max, int dtype) {
    if (B < 1 || Q < 1 || Hq < 1 || Hkv < 1 || d < 1 || L_max < 1) return 0;
    if (Hq % Hkv) return 0;
    if (dtype != 0 && dtype != 1) return 0;
    return 1;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Visible keys for query position qpos: vis = seq_len - Q + qpos + 1. */
static int visible(int seq_len, int Q, int qpos) { return seq_len - Q + qpos + 1; }

/* s[i] for i < vis of one row; returns vis (or -1 on a bad row). */
int oracle_row_scores(int B, int Q, int Hq, int Hkv, int d, int L_max, int dtype, double scale,
                      const void *q, const void *k_cache, const int32_t *seq_lens,
                      int b, int qpos, int h, double *s_out) {
    if (!check_shape(B, Q, Hq, Hkv, d, L_max, dtype)) return -1;
    if (b < 0 || b >= B || qpos < 0 || qpos >= Q || h < 0 || h >= Hq) return -1;
    int vis = visible(seq_lens[b], Q, qpos);
    if (seq_lens[b] > L_max || vis < 1) return -1;
    int G = Hq / Hkv, kvh = h / G;
    double sc = resolve_scale(scale, d);
    size_t qoff = (((size_t)b * Q + qpos) * Hq + h) * d;
    size_t koff = ((size_t)b * Hkv + kvh) * (size_t)L_max * d;
    for (int i = 0; i < vis; i++) {
        double acc = 0.0;
        for (int c = 0; c < d; c++)
            acc += load_elem(q, dtype, qoff + c) * load_elem(k_cache, dtype, koff + (size_t)i * d + c);
        s_out[i] = sc * acc;
    }
    return vis;
}

/*
 * Steps 3-6 for one row whose visible positions are already in (score
 * descending, position ascending) order in sp[0..vis): keep the first kk,
 * softmax over them, P.V, the discarded mass and the ascending idx (padded
 * with -1 up to idx_len).  sel is scratch of vis entries.
 */
static void attend_prefix(const scored_pos *sp, int vis, int kk, const void *v_cache, int dtype, size_t voff,
                          int d, double *o, double *tail_r, int32_t *ir, int idx_len, int32_t *sel) {
    double m = sp[0].s;
    double z_k = 0.0, z_tail = 0.0;
    for (int j = 0; j < kk; j++) z_k += exp(sp[j].s - m);
    for (int j = kk; j < vis; j++) z_tail += exp(sp[j].s - m);
    for (int c = 0; c < d; c++) o[c] = 0.0;
    for (int j = 0; j < kk; j++) {
        double p = exp(sp[j].s - m) / z_k;
        const size_t row = voff + (size_t)sp[j].i * d;
        for (int c = 0; c < d; c++) o[c] += p * load_elem(v_cache, dtype, row + c);
    }
    if (tail_r) *tail_r = z_tail / (z_k + z_tail);
    for (int j = 0; j < kk; j++) sel[j] = sp[j].i;
    qsort(sel, (size_t)kk, sizeof(int32_t), cmp_int_asc);
    for (int j = 0; j < idx_len; j++) ir[j] = j < kk ? sel[j] : -1;
}

/*
 * Token Top-k decode attention over all rows.
 *   out [B,Q,Hq,d], idx [B,Q,Hq,k], tail [B,Q,Hq], kth_score [B,Q,Hq] (the
 *   smallest kept score; -inf-free: equals the row minimum when k >= vis).
 *   tail and kth_score may be NULL.
 */
int oracle_topk_attn(int B, int Q, int Hq, int Hkv, int d, int L_max, int dtype, double scale,
                     const void *q, const void *k_cache, const void *v_cache, const int32_t *seq_lens,
                     int k, double *out, int32_t *idx, double *tail, double *kth_score, int nthreads) {
    if (!check_shape(B, Q, Hq, Hkv, d, L_max, dtype) || k < 1) return OR_BAD_ARG;
    for (int b = 0; b < B; b++)
        if (seq_lens[b] > L_max || visible(seq_lens[b], Q, 0) < 1) return OR_BAD_ARG;
    const int G = Hq / Hkv;
    const long rows = (long)B * Q * Hq;
    int status = OR_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        scored_pos *sp = (scored_pos *)malloc(sizeof(scored_pos) * (size_t)L_max);
        double *s = (double *)malloc(sizeof(double) * (size_t)L_max);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)L_max);
        if (!sp || !s || !sel) {
#pragma omp atomic write
            status = OR_NO_MEMORY;
        }
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < rows; r++) {
            if (!sp || !s || !sel) continue;
            int h = (int)(r % Hq), qpos = (int)((r / Hq) % Q), b = (int)(r / ((long)Hq * Q));
            int kvh = h / G;
            int vis = oracle_row_scores(B, Q, Hq, Hkv, d, L_max, dtype, scale, q, k_cache, seq_lens,
                                        b, qpos, h, s);
            /* 2. full stable order by (score desc, position asc) */
            for (int i = 0; i < vis; i++) { sp[i].s = s[i]; sp[i].i = i; }
            qsort(sp, (size_t)vis, sizeof(scored_pos), cmp_score_desc);
            int kk = k < vis ? k : vis;
            /* 3.-6. normalisers, P.V over the kept rows, discarded mass, idx */
            size_t voff = ((size_t)b * Hkv + kvh) * (size_t)L_max * d;
            attend_prefix(sp, vis, kk, v_cache, dtype, voff, d, out + (size_t)r * d, tail ? tail + r : NULL,
                          idx + (size_t)r * k, k, sel);
            if (kth_score) kth_score[r] = sp[kk - 1].s;
        }
        free(sp);
        free(s);
        free(sel);
    }
    return status;
}

/*
 * Certified adaptive Top-k ("A Mathematical Theory of Top-k Sparse Attention
 * via Total Variation Distance", abstract): the truncation error of Top-k
 * attention in total variation is the discarded softmax tail mass
 * tau_k = 1 - Z_k / Z, so the certified k of a row is the smallest k with
 * tau_k <= eps.  Per row, over the same (score descending, position
 * ascending) order as oracle_topk_attn:
 *   k_used = min{ k >= 1 : 1 - (sum_{j < k} e^{s_(j) - m}) / Z <= eps }, capped
 *   at min(k_max, vis) (when even that many keys leave more than eps outside,
 *   the cap is used and the returned tail exceeds eps);
 * then out, tail and idx exactly as oracle_topk_attn with k = k_used, idx
 * padded with -1 up to k_max.  k_used [B,Q,Hq] int32; tail may be NULL.
 */
int oracle_certified_attn(int B, int Q, int Hq, int Hkv, int d, int L_max, int dtype, double scale,
                          const void *q, const void *k_cache, const void *v_cache, const int32_t *seq_lens,
                          double eps, int k_max, double *out, int32_t *idx, double *tail, int32_t *k_used,
                          int nthreads) {
    if (!check_shape(B, Q, Hq, Hkv, d, L_max, dtype) || k_max < 1 || !(eps >= 0.0) || eps >= 1.0) return OR_BAD_ARG;
    for (int b = 0; b < B; b++)
        if (seq_lens[b] > L_max || visible(seq_lens[b], Q, 0) < 1) return OR_BAD_ARG;
    const int G = Hq / Hkv;
    const long rows = (long)B * Q * Hq;
    int status = OR_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        scored_pos *sp = (scored_pos *)malloc(sizeof(scored_pos) * (size_t)L_max);
        double *s = (double *)malloc(sizeof(double) * (size_t)L_max);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)L_max);
        if (!sp || !s || !sel) {
#pragma omp atomic write
            status = OR_NO_MEMORY;
        }
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < rows; r++) {
            if (!sp || !s || !sel) continue;
            int h = (int)(r % Hq), qpos = (int)((r / Hq) % Q), b = (int)(r / ((long)Hq * Q));
            int kvh = h / G;
            int vis = oracle_row_scores(B, Q, Hq, Hkv, d, L_max, dtype, scale, q, k_cache, seq_lens,
                                        b, qpos, h, s);
            for (int i = 0; i < vis; i++) { sp[i].s = s[i]; sp[i].i = i; }
            qsort(sp, (size_t)vis, sizeof(scored_pos), cmp_score_desc);
            double m = sp[0].s;
            double z = 0.0;
            for (int j = 0; j < vis; j++) z += exp(sp[j].s - m);
            /* the smallest prefix of the order whose discarded mass is <= eps */
            int cap = k_max < vis ? k_max : vis;
            int kk = cap;
            double z_k = 0.0;
            for (int j = 0; j < cap; j++) {
                z_k += exp(sp[j].s - m);
                if (1.0 - z_k / z <= eps) {
                    kk = j + 1;
                    break;
                }
            }
            size_t voff = ((size_t)b * Hkv + kvh) * (size_t)L_max * d;
            attend_prefix(sp, vis, kk, v_cache, dtype, voff, d, out + (size_t)r * d, tail ? tail + r : NULL,
                          idx + (size_t)r * k_max, k_max, sel);
            k_used[r] = kk;
        }
        free(sp);
        free(s);
        free(sel);
    }
    return status;
}

/*
 * MoBA block keys: block_keys[b, h, j, :] = mean of K[b, h, i, :] over the
 * tokens i of block j that lie below seq_len[b] (a partial last block is
 * averaged over the tokens it holds).  Blocks past the end are zero.
 * block_keys has shape [B, Hkv, ceil(L_max / block_size), d].
 */
int oracle_block_pool(int B, int Hkv, int d, int L_max, int dtype, const void *k_cache,
                      const int32_t *seq_lens, int block_size, double *block_keys) {
    if (B < 1 || Hkv < 1 || d < 1 || L_max < 1 || block_size < 1 || (dtype != 0 && dtype != 1))
        return OR_BAD_ARG;
    const int nblk_max = (L_max + block_size - 1) / block_size;
    for (int b = 0; b < B; b++) {
        if (seq_lens[b] < 1 || seq_lens[b] > L_max) return OR_BAD_ARG;
        for (int h = 0; h < Hkv; h++) {
            size_t koff = ((size_t)b * Hkv + h) * (size_t)L_max * d;
            double *bk = block_keys + ((size_t)b * Hkv + h) * (size_t)nblk_max * d;
            for (int j = 0; j < nblk_max; j++) {
                int lo = j * block_size, hi = lo + block_size;
                if (hi > seq_lens[b]) hi = seq_lens[b];
                for (int c = 0; c < d; c++) {
                    double acc = 0.0;
                    for (int i = lo; i < hi; i++) acc += load_elem(k_cache, dtype, koff + (size_t)i * d + c);
                    bk[(size_t)j * d + c] = hi > lo ? acc / (double)(hi - lo) : 0.0;
                }
            }
        }
    }
    return OR_OK;
}

/*
 * Block-sparse (MoBA) decode attention, one query position per sequence.
 *   out [B,Hq,d]; block_idx [B,Hq,top_blocks+1] ascending, -1 padded;
 *   tail [B,Hq] (nullable): softmax mass of the whole cache outside the kept
 *   blocks, for analysis; kth_block_score [B,Hq] (nullable): the smallest
 *   kept competing block score, or -HUGE_VAL when every block is kept.
 */
int oracle_block_attn(int B, int Hq, int Hkv, int d, int L_max, int dtype, double scale,
                      const void *q, const void *k_cache, const void *v_cache, const int32_t *seq_lens,
                      int block_size, int top_blocks, double *out, int32_t *block_idx,
                      double *tail, double *kth_block_score, int nthreads) {
    if (!check_shape(B, 1, Hq, Hkv, d, L_max, dtype) || block_size < 1 || top_blocks < 0)
        return OR_BAD_ARG;
    for (int b = 0; b < B; b++)
        if (seq_lens[b] < 1 || seq_lens[b] > L_max) return OR_BAD_ARG;
    const int G = Hq / Hkv;
    const int nblk_max = (L_max + block_size - 1) / block_size;
    double *bk = (double *)malloc(sizeof(double) * (size_t)B * Hkv * nblk_max * d);
    if (!bk) return OR_NO_MEMORY;
    int status = oracle_block_pool(B, Hkv, d, L_max, dtype, k_cache, seq_lens, block_size, bk);
    if (status != OR_OK) { free(bk); return status; }
    const double sc = resolve_scale(scale, d);
    const long rows = (long)B * Hq;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        scored_pos *sp = (scored_pos *)malloc(sizeof(scored_pos) * (size_t)nblk_max);
        double *s = (double *)malloc(sizeof(double) * (size_t)L_max);
        int32_t *kept = (int32_t *)malloc(sizeof(int32_t) * (size_t)(top_blocks + 1));
        char *in_sel = (char *)malloc((size_t)L_max);
        if (!sp || !s || !kept || !in_sel) {
#pragma omp atomic write
            status = OR_NO_MEMORY;
        }
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < rows; r++) {
            if (!sp || !s || !kept || !in_sel) continue;
            int h = (int)(r % Hq), b = (int)(r / Hq), kvh = h / G;
            int Lb = seq_lens[b];
            int nblk = (Lb + block_size - 1) / block_size;
            size_t qoff = (size_t)r * d;
            const double *bkh = bk + ((size_t)b * Hkv + kvh) * (size_t)nblk_max * d;
            /* block scores of the competing blocks j < nblk - 1 */
            for (int j = 0; j < nblk - 1; j++) {
                double acc = 0.0;
                for (int c = 0; c < d; c++) acc += load_elem(q, dtype, qoff + c) * bkh[(size_t)j * d + c];
                sp[j].s = sc * acc;
                sp[j].i = j;
            }
            qsort(sp, (size_t)(nblk - 1), sizeof(scored_pos), cmp_score_desc);
            int nk = top_blocks < nblk - 1 ? top_blocks : nblk - 1;
            for (int j = 0; j < nk; j++) kept[j] = sp[j].i;
            kept[nk] = nblk - 1; /* the current block */
            if (kth_block_score) kth_block_score[r] = nk > 0 && nk < nblk - 1 ? sp[nk - 1].s : -HUGE_VAL;
            qsort(kept, (size_t)(nk + 1), sizeof(int32_t), cmp_int_asc);
            int32_t *bi = block_idx + (size_t)r * (top_blocks + 1);
            for (int j = 0; j <= top_blocks; j++) bi[j] = j <= nk ? kept[j] : -1;
            /* dense softmax attention over the tokens of the kept blocks */
            memset(in_sel, 0, (size_t)Lb);
            for (int j = 0; j <= nk; j++) {
                int lo = kept[j] * block_size, hi = lo + block_size;
                if (hi > Lb) hi = Lb;
                for (int i = lo; i < hi; i++) in_sel[i] = 1;
            }
            oracle_row_scores(B, 1, Hq, Hkv, d, L_max, dtype, scale, q, k_cache, seq_lens, b, 0, h, s);
            double m = -HUGE_VAL, m_all = -HUGE_VAL;
            for (int i = 0; i < Lb; i++) {
                if (s[i] > m_all) m_all = s[i];
                if (in_sel[i] && s[i] > m) m = s[i];
            }
            double z = 0.0, z_out = 0.0, z_all = 0.0;
            for (int i = 0; i < Lb; i++) {
                z_all += exp(s[i] - m_all);
                if (in_sel[i]) z += exp(s[i] - m);
                else z_out += exp(s[i] - m_all);
            }
            double *o = out + (size_t)r * d;
            for (int c = 0; c < d; c++) o[c] = 0.0;
            size_t voff = ((size_t)b * Hkv + kvh) * (size_t)L_max * d;
            for (int i = 0; i < Lb; i++) {
                if (!in_sel[i]) continue;
                double p = exp(s[i] - m) / z;
                for (int c = 0; c < d; c++) o[c] += p * load_elem(v_cache, dtype, voff + (size_t)i * d + c);
            }
            if (tail) tail[r] = z_out / z_all;
        }
        free(sp);
        free(s);
        free(kept);
        free(in_sel);
    }
    free(bk);
    return status;
}

/*
 * Hierarchical block -> token selection ("Sparse Attention Landscape",
 * section "Hierarchical Sparse Attention"), one query per sequence:
 *   1. block scores r_j = scale * <q, mean key of block j> for every block j
 *      of the sequence (the partial last block averaged over its tokens);
 *   2. the top_blocks best blocks (r descending, block ascending) are kept;
 *   3. token scores s_i = scale * <q, K_i> only for the tokens of the kept
 *      blocks below seq_len (the candidates);
 *   4. the top k candidates (s descending, position ascending) are kept and
 *      attention runs over them: softmax over the kept tokens, P.V;
 *   5. tail = the candidates' discarded softmax mass, relative to all
 *      candidates (the method scores nothing else).
 * block_idx [B, Hq, top_blocks] and idx [B, Hq, k] ascending, -1 padded.
 */
int oracle_hisa_attn(int B, int Hq, int Hkv, int d, int L_max, int dtype, double scale,
                     const void *q, const void *k_cache, const void *v_cache, const int32_t *seq_lens,
                     int block_size, int top_blocks, int k, double *out, int32_t *block_idx, int32_t *idx,
                     double *tail, int nthreads) {
    if (!check_shape(B, 1, Hq, Hkv, d, L_max, dtype) || block_size < 1 || top_blocks < 1 || k < 1)
        return OR_BAD_ARG;
    for (int b = 0; b < B; b++)
        if (seq_lens[b] < 1 || seq_lens[b] > L_max) return OR_BAD_ARG;
    const int G = Hq / Hkv;
    const int nblk_max = (L_max + block_size - 1) / block_size;
    double *bk = (double *)malloc(sizeof(double) * (size_t)B * Hkv * nblk_max * d);
    if (!bk) return OR_NO_MEMORY;
    int status = oracle_block_pool(B, Hkv, d, L_max, dtype, k_cache, seq_lens, block_size, bk);
    if (status != OR_OK) { free(bk); return status; }
    const double sc = resolve_scale(scale, d);
    const long rows = (long)B * Hq;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        scored_pos *sb = (scored_pos *)malloc(sizeof(scored_pos) * (size_t)nblk_max);
        scored_pos *sp = (scored_pos *)malloc(sizeof(scored_pos) * (size_t)L_max);
        double *s = (double *)malloc(sizeof(double) * (size_t)L_max);
        int32_t *kept = (int32_t *)malloc(sizeof(int32_t) * (size_t)nblk_max);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)L_max);
        if (!sb || !sp || !s || !kept || !sel) {
#pragma omp atomic write
            status = OR_NO_MEMORY;
        }
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < rows; r++) {
            if (!sb || !sp || !s || !kept || !sel) continue;
            int h = (int)(r % Hq), b = (int)(r / Hq), kvh = h / G;
            int Lb = seq_lens[b];
            int nblk = (Lb + block_size - 1) / block_size;
            size_t qoff = (size_t)r * d;
            const double *bkh = bk + ((size_t)b * Hkv + kvh) * (size_t)nblk_max * d;
            /* 1.-2. block scores of every block, the best top_blocks kept */
            for (int j = 0; j < nblk; j++) {
                double acc = 0.0;
                for (int c = 0; c < d; c++) acc += load_elem(q, dtype, qoff + c) * bkh[(size_t)j * d + c];
                sb[j].s = sc * acc;
                sb[j].i = j;
            }
            qsort(sb, (size_t)nblk, sizeof(scored_pos), cmp_score_desc);
            int nk = top_blocks < nblk ? top_blocks : nblk;
            for (int j = 0; j < nk; j++) kept[j] = sb[j].i;
            qsort(kept, (size_t)nk, sizeof(int32_t), cmp_int_asc);
            int32_t *bi = block_idx + (size_t)r * top_blocks;
            for (int j = 0; j < top_blocks; j++) bi[j] = j < nk ? kept[j] : -1;
            /* 3. token scores of the candidates, in position order */
            oracle_row_scores(B, 1, Hq, Hkv, d, L_max, dtype, scale, q, k_cache, seq_lens, b, 0, h, s);
            int nc = 0;
            for (int j = 0; j < nk; j++) {
                int lo = kept[j] * block_size, hi = lo + block_size;
                if (hi > Lb) hi = Lb;
                for (int i = lo; i < hi; i++) {
                    sp[nc].s = s[i];
                    sp[nc].i = i;
                    nc++;
                }
            }
            /* 4.-5. top k of the candidates, attention over them, discarded candidate mass */
            qsort(sp, (size_t)nc, sizeof(scored_pos), cmp_score_desc);
            int kk = k < nc ? k : nc;
            size_t voff = ((size_t)b * Hkv + kvh) * (size_t)L_max * d;
            attend_prefix(sp, nc, kk, v_cache, dtype, voff, d, out + (size_t)r * d, tail ? tail + r : NULL,
                          idx + (size_t)r * k, k, sel);
        }
        free(sb);
        free(sp);
        free(s);
        free(kept);
        free(sel);
    }
    free(bk);
    return status;
}

/*
 * Token selection by a lightning indexer ("Sparse Attention Landscape",
 * section "Token Sparse Attention", DeepSeek Sparse Attention): the indexer
 * scores every visible token of a query position with its own small heads,
 *   I_i = sum_j w[j] * ReLU(<q_idx[j], k_idx[i]>),   j < H_I,
 * where q_idx [B, Q, H_I, d_I], w_idx [B, Q, H_I] (fp32) and k_idx
 * [B, L_max, d_I] are the indexer's projected queries, head weights and keys
 * (inputs here); the top k tokens by I (descending, position ascending) are
 * kept for the query position, shared by all attention heads; then every
 * head h attends over them with its exact scores:
 *   out = sum_{i kept} softmax_i(scale * <q_h, K[b, h / G, i, :]>) V[b, h / G, i, :].
 * idx [B, Q, k] ascending, -1 padded; kth_index [B, Q] the smallest kept I.
 */
int oracle_indexer_attn(int B, int Q, int Hq, int Hkv, int d, int L_max, int dtype, double scale,
                        const void *q, const void *k_cache, const void *v_cache, const int32_t *seq_lens,
                        int H_I, int d_I, const void *q_idx, const float *w_idx, const void *k_idx, int k,
                        double *out, int32_t *idx, double *kth_index, int nthreads) {
    if (!check_shape(B, Q, Hq, Hkv, d, L_max, dtype) || H_I < 1 || d_I < 1 || k < 1) return OR_BAD_ARG;
    for (int b = 0; b < B; b++)
        if (seq_lens[b] > L_max || visible(seq_lens[b], Q, 0) < 1) return OR_BAD_ARG;
    const int G = Hq / Hkv;
    const long units = (long)B * Q;
    int status = OR_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        scored_pos *sp = (scored_pos *)malloc(sizeof(scored_pos) * (size_t)L_max);
        scored_pos *kept = (scored_pos *)malloc(sizeof(scored_pos) * (size_t)L_max);
        double *s = (double *)malloc(sizeof(double) * (size_t)L_max);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * 2 * (size_t)L_max);  /* kept positions + scratch */
        if (!sp || !kept || !s || !sel) {
#pragma omp atomic write
            status = OR_NO_MEMORY;
        }
#pragma omp for schedule(dynamic, 1)
        for (long u = 0; u < units; u++) {
            if (!sp || !kept || !s || !sel) continue;
            int qpos = (int)(u % Q), b = (int)(u / Q);
            int vis = visible(seq_lens[b], Q, qpos);
            /* indexer scores of every visible token */
            for (int i = 0; i < vis; i++) {
                double acc = 0.0;
                for (int j = 0; j < H_I; j++) {
                    double dot = 0.0;
                    size_t qo = ((size_t)u * H_I + j) * d_I, ko = ((size_t)b * L_max + i) * d_I;
                    for (int c = 0; c < d_I; c++) dot += load_elem(q_idx, dtype, qo + c) * load_elem(k_idx, dtype, ko + c);
                    acc += (double)w_idx[(size_t)u * H_I + j] * (dot > 0.0 ? dot : 0.0);
                }
                sp[i].s = acc;
                sp[i].i = i;
            }
            qsort(sp, (size_t)vis, sizeof(scored_pos), cmp_score_desc);
            int kk = k < vis ? k : vis;
            if (kth_index) kth_index[u] = sp[kk - 1].s;
            for (int j = 0; j < kk; j++) sel[j] = sp[j].i;
            qsort(sel, (size_t)kk, sizeof(int32_t), cmp_int_asc);
            int32_t *ir = idx + (size_t)u * k;
            for (int j = 0; j < k; j++) ir[j] = j < kk ? sel[j] : -1;
            /* every head attends over the kept tokens with its exact scores */
            for (int h = 0; h < Hq; h++) {
                int kvh = h / G;
                oracle_row_scores(B, Q, Hq, Hkv, d, L_max, dtype, scale, q, k_cache, seq_lens, b, qpos, h, s);
                for (int j = 0; j < kk; j++) {
                    kept[j].s = s[sel[j]];
                    kept[j].i = sel[j];
                }
                qsort(kept, (size_t)kk, sizeof(scored_pos), cmp_score_desc);
                size_t voff = ((size_t)b * Hkv + kvh) * (size_t)L_max * d;
                size_t r = (size_t)u * Hq + h;
                attend_prefix(kept, kk, kk, v_cache, dtype, voff, d, out + r * d, NULL, sel + kk, 0, sel + kk);
            }
        }
        free(sp);
        free(kept);
        free(s);
        free(sel);
    }
    return status;
}
