/*
 * sa_oracle.c -- plain, slow, double-precision CPU oracle for sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header or table with the CUDA library.
 *
 * What it computes (sources are the web pages collected on sparse attention):
 *
 *  - "Sparse Attention Weights Assumption" (1cademy), sparse attention output
 *    formula: out_i = sum_{j in G_i} alpha'_{i,j} v_j with G_i a subset of
 *    {0..i} for a causal model.  alpha' is read as the softmax of the scaled
 *    logits restricted to G_i (renormalised over G_i), the only reading under
 *    which a full G reproduces the dense formula below.
 *  - "sparse attention mechanism" glossary (chipfoundryservices), "Standard
 *    Attention Bottleneck": Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V.
 *  - same glossary, "Sparse Attention Patterns" table and "Mistral/Mixtral
 *    Sliding Window Attention": sliding window [max(0, i-W+1), i] (causal),
 *    w nearest neighbours (non-causal, read as |i-j| <= W/2), global tokens,
 *    BigBird random blocks, blockwise (block-local) attention; and
 *    "Multi-Query and Grouped-Query Attention": H query heads share H_kv K/V
 *    heads (read as contiguous groups, h_kv = h / (H / H_kv)).
 *    The same table's dilated/strided row ("every k-th token", O(N*w)) is read
 *    as the window with its taps k apart: (i - j) mod k == 0 and the window
 *    test applied to the tap number m = (i - j) / k.
 *  - "SAS: Sparse Attention Synthesizer" (kindchill), Step 5 component 1,
 *    primitive C ("attend to top-K dynamic tokens"), and the dynamic patterns
 *    of "Sparse Attention Weights Assumption" (tokens with the highest
 *    relevance scores): for one decode query, G = the top_k keys by relevance
 *    score s_j = scale * q . k_j, ties to the smaller index (ora_topk_select);
 *    the output is then the sparse output formula over that G.
 *  - "SAS: Sparse Attention Synthesizer" (kindchill), Step 5 component 2:
 *    patterns are combined from primitives by logical OR.
 *  - "Block Sparse Flash Attention" (montaan AI Radio), paper summary and
 *    improvements: the exact QK^T scores of a key block are computed, the
 *    block's maximum is compared with a per-(layer, head) calibrated threshold,
 *    and the block's PV product and V load are skipped below it.  Read here as:
 *    one decision per (query tile, key block); the statistic is the maximum
 *    scaled logit over the tile's visible pairs; only blocks whose every pair
 *    is visible ("full" blocks) may be skipped; a skipped block's keys leave
 *    G_i for every row i of the tile (so they leave the softmax denominator).
 *    The episode's summary words the rule per query (each query's scores
 *    decide which value blocks matter); that reading is built as an option:
 *    a row also drops a full block when its own maximum over the block is
 *    below the threshold, and the block is skipped when every row drops it.
 *
 * Steps follow the definitions in order: build G_i explicitly, compute logits
 * for j in G_i, max, exp, sum, normalise, weighted sum of V rows.  Two passes,
 * no online softmax, no tiling of the arithmetic.  exp/log come from libm.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t causal;        /* 1: j <= i                                            */
    int32_t window;        /* 0 off; causal: j in [i-W+1, i]; else |i-j| <= W/2    */
    int32_t n_global;      /* 0 off; tokens 0..g-1 are seen by all and see all     */
    int32_t block_local;   /* 0 off; i and j in the same block of this size        */
    int32_t block_q;       /* query-tile height used by the block-skip rule        */
    int32_t block_k;       /* key-block width used by the block-skip rule          */
    int32_t random_block;  /* granularity of random blocks (rows and keys)         */
    int32_t n_random;      /* random key blocks per (head, query block)            */
    const int32_t *random_table; /* [H][ceil(N/random_block)][n_random] or NULL   */
    int32_t dilation;      /* window taps this far apart; 0 or 1: contiguous       */
} ora_pattern_t;

static int dilation_of(const ora_pattern_t *p) { return p->dilation > 1 ? p->dilation : 1; }

/* Inputs are either raw bf16 bit patterns (kind 0), converted exactly to
 * double, or doubles (kind 1). */
static double ld(const void *base, int64_t idx, int kind)
{
    if (kind == 0) {
        uint32_t u = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return ((const double *)base)[idx];
}

static int random_on(const ora_pattern_t *p)
{
    return p->n_random > 0 && p->random_table != NULL && p->random_block > 0;
}

/* ---- membership of (i, j) in G_i, written straight from the definitions ---- */
int ora_visible(const ora_pattern_t *p, int N, int h, int i, int j)
{
    if (i < 0 || i >= N || j < 0 || j >= N) return 0;
    if (p->causal && j > i) return 0;
    int any_primitive = 0, in = 0;
    if (p->window > 0) {
        any_primitive = 1;
        int k = dilation_of(p);
        int dist = i - j;
        if (dist % k == 0) {              /* j is one of the window's taps */
            int m = dist / k;             /* tap number, 0 = the query itself */
            if (p->causal) {
                if (m >= 0 && m <= p->window - 1) in = 1;
            } else {
                if (abs(m) <= p->window / 2) in = 1;
            }
        }
    }
    if (p->n_global > 0) {
        any_primitive = 1;
        if (i < p->n_global || j < p->n_global) in = 1;
    }
    if (p->block_local > 0) {
        any_primitive = 1;
        if (i / p->block_local == j / p->block_local) in = 1;
    }
    if (random_on(p)) {
        any_primitive = 1;
        int nrb = (N + p->random_block - 1) / p->random_block;
        const int32_t *row = p->random_table +
            ((int64_t)h * nrb + i / p->random_block) * p->n_random;
        for (int r = 0; r < p->n_random; ++r)
            if (row[r] == j / p->random_block) in = 1;
    }
    return any_primitive ? in : 1;
}

/* ---- G_i built a second way: as a union of index ranges ---- */
typedef struct { int64_t lo, hi; } range_t;   /* [lo, hi) */

static int cmp_range(const void *a, const void *b)
{
    const range_t *x = (const range_t *)a, *y = (const range_t *)b;
    return (x->lo > y->lo) - (x->lo < y->lo);
}

/* Writes the sorted members of G_i to out (capacity N); returns |G_i|. */
int ora_build_G(const ora_pattern_t *p, int N, int h, int i, int32_t *out)
{
    int cap = 4 + (random_on(p) ? p->n_random : 0);
    range_t *r = (range_t *)malloc(sizeof(range_t) * cap);
    int nr = 0, any_primitive = 0;
    int dilated = p->window > 0 && dilation_of(p) > 1;   /* taps merged in below */
    if (dilated) any_primitive = 1;
    if (p->window > 0 && !dilated) {
        any_primitive = 1;
        if (p->causal) { r[nr].lo = (int64_t)i - p->window + 1; r[nr].hi = (int64_t)i + 1; }
        else           { r[nr].lo = (int64_t)i - p->window / 2; r[nr].hi = (int64_t)i + p->window / 2 + 1; }
        nr++;
    }
    if (p->n_global > 0) {
        any_primitive = 1;
        if (i < p->n_global) { r[nr].lo = 0; r[nr].hi = N; }
        else                 { r[nr].lo = 0; r[nr].hi = p->n_global; }
        nr++;
    }
    if (p->block_local > 0) {
        any_primitive = 1;
        r[nr].lo = (int64_t)(i / p->block_local) * p->block_local;
        r[nr].hi = r[nr].lo + p->block_local;
        nr++;
    }
    if (random_on(p)) {
        any_primitive = 1;
        int nrb = (N + p->random_block - 1) / p->random_block;
        const int32_t *row = p->random_table +
            ((int64_t)h * nrb + i / p->random_block) * p->n_random;
        for (int k = 0; k < p->n_random; ++k) {
            r[nr].lo = (int64_t)row[k] * p->random_block;
            r[nr].hi = r[nr].lo + p->random_block;
            nr++;
        }
    }
    if (!any_primitive) { r[0].lo = 0; r[0].hi = N; nr = 1; }

    int64_t cap_hi = p->causal ? (int64_t)i + 1 : (int64_t)N;
    if (cap_hi > N) cap_hi = N;
    qsort(r, nr, sizeof(range_t), cmp_range);
    int n = 0;
    int64_t next = 0;               /* first index not yet emitted */
    for (int k = 0; k < nr; ++k) {
        int64_t lo = r[k].lo < next ? next : r[k].lo;
        if (lo < 0) lo = 0;
        int64_t hi = r[k].hi < cap_hi ? r[k].hi : cap_hi;
        for (int64_t j = lo; j < hi; ++j) out[n++] = (int32_t)j;
        if (hi > next) next = hi;
    }
    free(r);
    if (dilated) {
        /* the window's taps i + m*k, listed in ascending order, merged with the
           (sorted, distinct) members emitted above */
        int64_t k = dilation_of(p);
        int64_t m_lo = p->causal ? -(int64_t)(p->window - 1) : -(int64_t)(p->window / 2);
        int64_t m_hi = p->causal ? 0 : (int64_t)(p->window / 2);
        int32_t *taps = (int32_t *)malloc(sizeof(int32_t) * (size_t)(m_hi - m_lo + 1));
        int nt = 0;
        for (int64_t m = m_lo; m <= m_hi; ++m) {
            int64_t j = (int64_t)i + m * k;
            if (j >= 0 && j < cap_hi) taps[nt++] = (int32_t)j;
        }
        int32_t *merged = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + nt + 1));
        int a = 0, b = 0, c = 0;
        while (a < n || b < nt) {
            int32_t v;
            if (b >= nt || (a < n && out[a] <= taps[b])) v = out[a++];
            else v = taps[b++];
            if (c == 0 || merged[c - 1] != v) merged[c++] = v;
        }
        memcpy(out, merged, sizeof(int32_t) * (size_t)c);
        n = c;
        free(merged);
        free(taps);
    }
    return n;
}

/* ---- the weighted sum of the sparse output formula: out = sum_k alpha[k] v_{G[k]} ----
 * Shared by every entry point below, so the worked-example pin exercises the
 * same final step that the prefill and gather rows use. */
static void weighted_sum_rows(int kind, const void *V, int64_t kv_off, int d,
                              const int32_t *G, int nG, const double *alpha, double *out)
{
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    for (int k = 0; k < nG; ++k) {
        int64_t vrow = kv_off + (int64_t)G[k] * d;
        for (int c = 0; c < d; ++c) out[c] += alpha[k] * ld(V, vrow + c, kind);
    }
}

void ora_weighted_sum(int nG, int d, const int32_t *G, const double *alpha,
                      const double *V, double *out)
{
    weighted_sum_rows(1, V, 0, d, G, nG, alpha, out);
}

/* One query row over an explicit index list G (plain two-pass softmax).
 * q_off / kv_off are element offsets of the row q and of key/value row 0.
 * extra_w lists logits that enter the denominator only (used by the
 * keep-in-denominator variant of the block-skip rule).  Empty G -> out = 0,
 * lse = -inf. */
static void row_attention(int kind, const void *Q, int64_t q_off,
                          const void *K, const void *V, int64_t kv_off,
                          int d, double scale, const int32_t *G, int nG,
                          const double *extra_s, int n_extra,
                          double *out, double *lse)
{
    if (nG == 0 && n_extra == 0) {
        for (int c = 0; c < d; ++c) out[c] = 0.0;
        *lse = -INFINITY;
        return;
    }
    /* with nG == 0 but denominator-only terms, out = 0 and lse is theirs */
    double *s = (double *)malloc(sizeof(double) * (size_t)(nG > 0 ? nG : 1));
    double m = -INFINITY;
    for (int k = 0; k < nG; ++k) {
        double acc = 0.0;
        int64_t krow = kv_off + (int64_t)G[k] * d;
        for (int c = 0; c < d; ++c) acc += ld(Q, q_off + c, kind) * ld(K, krow + c, kind);
        s[k] = scale * acc;
        if (s[k] > m) m = s[k];
    }
    for (int k = 0; k < n_extra; ++k) if (extra_s[k] > m) m = extra_s[k];
    double l = 0.0;
    for (int k = 0; k < nG; ++k) { s[k] = exp(s[k] - m); l += s[k]; }
    for (int k = 0; k < n_extra; ++k) l += exp(extra_s[k] - m);
    for (int k = 0; k < nG; ++k) s[k] /= l;          /* alpha'_{i,j} */
    weighted_sum_rows(kind, V, kv_off, d, G, nG, s, out);
    *lse = m + log(l);
    free(s);
}

/* ---- block-skip rule for one query tile (b, h, t) ----
 * For every key block kb: cnt = number of (i, j) pairs of the tile with
 * j in G_i (static pattern) and j in block kb; full = (cnt == block_q*block_k);
 * stat = max over those pairs of scale * q_i . k_j; skip = full && stat < tau
 * (strict) unless override[kb] >= 0 forces keep (0) or skip (1).
 * mask: 0 = no pair, 1 = computed and kept, 2 = skipped.  Arrays have n_kb. */
void ora_tile_blocks(const ora_pattern_t *p, int kind, int B, int H, int Hkv,
                     int N, int d, double scale, const void *Q, const void *K,
                     int b, int h, int t, const double *thresholds,
                     const int8_t *override_kb, int64_t *cnt, uint8_t *full,
                     double *stat, uint8_t *mask)
{
    (void)B;
    int n_kb = (N + p->block_k - 1) / p->block_k;
    int hkv = h / (H / Hkv);
    for (int kb = 0; kb < n_kb; ++kb) { cnt[kb] = 0; stat[kb] = -INFINITY; }
    int32_t *G = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    int i0 = t * p->block_q, i1 = i0 + p->block_q;
    if (i1 > N) i1 = N;
    for (int i = i0; i < i1; ++i) {
        int nG = ora_build_G(p, N, h, i, G);
        int64_t q_off = (((int64_t)b * H + h) * N + i) * d;
        for (int k = 0; k < nG; ++k) {
            int j = G[k];
            int64_t k_off = (((int64_t)b * Hkv + hkv) * N + j) * d;
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += ld(Q, q_off + c, kind) * ld(K, k_off + c, kind);
            double s = scale * acc;
            int kb = j / p->block_k;
            cnt[kb]++;
            if (s > stat[kb]) stat[kb] = s;
        }
    }
    free(G);
    for (int kb = 0; kb < n_kb; ++kb) {
        full[kb] = cnt[kb] == (int64_t)p->block_q * p->block_k;
        int skip = 0;
        if (thresholds != NULL && full[kb] && stat[kb] < thresholds[h]) skip = 1;
        if (override_kb != NULL && override_kb[kb] >= 0) skip = override_kb[kb] ? 1 : 0;
        mask[kb] = cnt[kb] == 0 ? 0 : (skip ? 2 : 1);
    }
}

/* ---- prefill: rows (b, h, i) of out_i = sum_{j in G_i} softmax_G(s_ij) v_j ----
 * rows: n_rows triplets (b, h, i), or NULL for every row in [B][H][N] order.
 * thresholds: [H] block-skip thresholds in scaled-logit units, or NULL (off).
 * override: [B][H][T][n_kb] int8 (-1 = rule, 0 = keep, 1 = skip) or NULL.
 * keep_in_denominator: 1 = skipped keys' logits still enter the denominator
 *   (the variant reading; not the default).
 * row_level: 1 = the per-query reading of the rule ("Block Sparse Flash
 *   Attention", paper summary: the scores of each query decide which value
 *   blocks matter): on top of the tile decisions, row i drops a full block of
 *   its tile from G_i when its own maximum scaled logit over the block's keys
 *   is below the threshold.  A tile's block is skipped (mask 2) exactly when
 *   every row drops it, which is the tile rule's decision; partial blocks are
 *   never dropped.  Not combined with keep_in_denominator.
 * row_override: [n_rows][n_kb] int8 (-1 = rule, 0 = keep, 1 = drop) or NULL,
 *   per requested row and key block (row_level only).
 * row_stat_out: [n_rows][n_kb] (nullable, row_level only): the row's maximum
 *   scaled logit over each full block of its tile, -inf for other blocks.
 * mask_out / stat_out / full_out: [B][H][T][n_kb] (nullable); only tiles
 *   that hold a requested row are written.  O: [n_rows][d], lse: [n_rows]. */
void ora_prefill(const ora_pattern_t *p, int kind, int B, int H, int Hkv, int N,
                 int d, double scale, const void *Q, const void *K, const void *V,
                 const double *thresholds, const int8_t *override_mask,
                 int keep_in_denominator, int row_level, const int8_t *row_override,
                 double *row_stat_out, int64_t n_rows, const int32_t *rows,
                 double *O, double *lse, uint8_t *mask_out, double *stat_out,
                 uint8_t *full_out, int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int T = (N + p->block_q - 1) / p->block_q;
    int n_kb = (N + p->block_k - 1) / p->block_k;
    int64_t total = rows ? n_rows : (int64_t)B * H * N;
    int need_tiles = thresholds != NULL || override_mask != NULL ||
                     mask_out != NULL || stat_out != NULL || full_out != NULL;

    /* 1. which tiles hold a requested row */
    uint8_t *tile_needed = NULL;
    uint8_t *tile_mask = NULL;     /* [B*H*T][n_kb] decisions */
    double *tile_stat = NULL;
    int64_t *tile_cnt = NULL;
    if (need_tiles) {
        tile_needed = (uint8_t *)calloc((size_t)B * H * T, 1);
        for (int64_t r = 0; r < total; ++r) {
            int b, h, i;
            if (rows) { b = rows[3 * r]; h = rows[3 * r + 1]; i = rows[3 * r + 2]; }
            else { b = (int)(r / ((int64_t)H * N)); h = (int)((r / N) % H); i = (int)(r % N); }
            tile_needed[((int64_t)b * H + h) * T + i / p->block_q] = 1;
        }
        tile_mask = (uint8_t *)calloc((size_t)B * H * T * n_kb, 1);
        tile_stat = (double *)malloc(sizeof(double) * (size_t)B * H * T * n_kb);
        tile_cnt = (int64_t *)malloc(sizeof(int64_t) * (size_t)B * H * T * n_kb);
        uint8_t *full_all = (uint8_t *)malloc((size_t)B * H * T * n_kb);
        /* 2. block decisions for every needed tile */
        #pragma omp parallel for schedule(dynamic, 1)
        for (int64_t u = 0; u < (int64_t)B * H * T; ++u) {
            if (!tile_needed[u]) continue;
            int b = (int)(u / ((int64_t)H * T)), h = (int)((u / T) % H), t = (int)(u % T);
            ora_tile_blocks(p, kind, B, H, Hkv, N, d, scale, Q, K, b, h, t,
                            thresholds, override_mask ? override_mask + u * n_kb : NULL,
                            tile_cnt + u * n_kb, full_all + u * n_kb,
                            tile_stat + u * n_kb, tile_mask + u * n_kb);
        }
        for (int64_t u = 0; u < (int64_t)B * H * T; ++u) {
            if (!tile_needed[u]) continue;
            for (int kb = 0; kb < n_kb; ++kb) {
                if (mask_out) mask_out[u * n_kb + kb] = tile_mask[u * n_kb + kb];
                if (stat_out) stat_out[u * n_kb + kb] = tile_stat[u * n_kb + kb];
                if (full_out) full_out[u * n_kb + kb] = full_all[u * n_kb + kb];
            }
        }
        free(full_all);
    }

    /* 3. every requested row */
    #pragma omp parallel
    {
        int32_t *G = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
        int32_t *Gk = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
        double *extra = (double *)malloc(sizeof(double) * (size_t)N);
        double *rmax = (double *)malloc(sizeof(double) * (size_t)n_kb);
        uint8_t *rdrop = (uint8_t *)malloc((size_t)n_kb);
        #pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < total; ++r) {
            int b, h, i;
            if (rows) { b = rows[3 * r]; h = rows[3 * r + 1]; i = rows[3 * r + 2]; }
            else { b = (int)(r / ((int64_t)H * N)); h = (int)((r / N) % H); i = (int)(r % N); }
            int hkv = h / (H / Hkv);
            int nG = ora_build_G(p, N, h, i, G);
            int nk = 0, ne = 0;
            int64_t q_off = (((int64_t)b * H + h) * N + i) * d;
            int64_t kv_off = ((int64_t)b * Hkv + hkv) * N * d;
            int64_t u_row = ((int64_t)b * H + h) * T + i / p->block_q;
            const uint8_t *tm = need_tiles ? tile_mask + u_row * n_kb : NULL;
            if (row_level && thresholds != NULL) {
                /* the row's own maximum over each full block of its tile */
                const int64_t *tc = tile_cnt + u_row * n_kb;
                for (int kb = 0; kb < n_kb; ++kb) rmax[kb] = -INFINITY;
                for (int k = 0; k < nG; ++k) {
                    int j = G[k], kb = j / p->block_k;
                    if (tc[kb] != (int64_t)p->block_q * p->block_k) continue;
                    double acc = 0.0;
                    for (int c = 0; c < d; ++c)
                        acc += ld(Q, q_off + c, kind) * ld(K, kv_off + (int64_t)j * d + c, kind);
                    if (scale * acc > rmax[kb]) rmax[kb] = scale * acc;
                }
                for (int kb = 0; kb < n_kb; ++kb) {
                    int full = tc[kb] == (int64_t)p->block_q * p->block_k;
                    int drop = full && rmax[kb] < thresholds[h];
                    if (row_override != NULL && row_override[r * n_kb + kb] >= 0)
                        drop = row_override[r * n_kb + kb] ? 1 : 0;
                    rdrop[kb] = (uint8_t)drop;
                    if (row_stat_out) row_stat_out[r * n_kb + kb] = full ? rmax[kb] : -INFINITY;
                }
            }
            for (int k = 0; k < nG; ++k) {
                int j = G[k];
                if (row_level && thresholds != NULL && tm && tm[j / p->block_k] != 2 &&
                    rdrop[j / p->block_k])
                    continue;   /* dropped by this row alone: the key leaves G_i */
                if (tm && tm[j / p->block_k] == 2) {
                    if (keep_in_denominator) {
                        double acc = 0.0;
                        for (int c = 0; c < d; ++c)
                            acc += ld(Q, q_off + c, kind) * ld(K, kv_off + (int64_t)j * d + c, kind);
                        extra[ne++] = scale * acc;
                    }
                    continue;
                }
                Gk[nk++] = j;
            }
            row_attention(kind, Q, q_off, K, V, kv_off, d, scale, Gk, nk, extra, ne,
                          O + r * d, lse + r);
        }
        free(G); free(Gk); free(extra); free(rmax); free(rdrop);
    }
    free(tile_needed); free(tile_mask); free(tile_stat); free(tile_cnt);
}

/* ---- dense attention in matrix form: softmax(Q K^T * scale [+ causal mask]) V ----
 * A separate routine (full score matrix per head) used only to pin the
 * sparse path: a full G must reproduce it.  O: [B][H][N][d]. */
void ora_dense(int kind, int B, int H, int Hkv, int N, int d, double scale,
               int causal, const void *Q, const void *K, const void *V, double *O)
{
    double *S = (double *)malloc(sizeof(double) * (size_t)N * N);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            int hkv = h / (H / Hkv);
            int64_t qb = ((int64_t)b * H + h) * N * d, kvb = ((int64_t)b * Hkv + hkv) * N * d;
            for (int i = 0; i < N; ++i)
                for (int j = 0; j < N; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < d; ++c)
                        acc += ld(Q, qb + (int64_t)i * d + c, kind) * ld(K, kvb + (int64_t)j * d + c, kind);
                    S[(int64_t)i * N + j] = (causal && j > i) ? -INFINITY : scale * acc;
                }
            for (int i = 0; i < N; ++i) {
                double *row = S + (int64_t)i * N, m = -INFINITY, l = 0.0;
                for (int j = 0; j < N; ++j) if (row[j] > m) m = row[j];
                for (int j = 0; j < N; ++j) { row[j] = exp(row[j] - m); l += row[j]; }
                for (int j = 0; j < N; ++j) row[j] /= l;
            }
            for (int i = 0; i < N; ++i)
                for (int c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < N; ++j)
                        acc += S[(int64_t)i * N + j] * ld(V, kvb + (int64_t)j * d + c, kind);
                    O[qb + (int64_t)i * d + c] = acc;
                }
        }
    free(S);
}

/* ---- explicit index sets over a KV cache (decode) ----
 * Q, O: [S][H][d]; K, V: [S][Hkv][L][d]; idx: [S][H_idx][n_idx] (each set
 * sorted and unique); idx_len: [S][H_idx] or NULL (= n_idx).  H_idx is H (one
 * set per query head) or Hkv (one set per K/V head, shared by its group). */
void ora_gather(int kind, int S, int H, int Hkv, int H_idx, int L, int d, int n_idx,
                double scale, const void *Q, const void *K, const void *V,
                const int32_t *idx, const int32_t *idx_len, double *O, double *lse,
                int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < (int64_t)S * H; ++u) {
        int s = (int)(u / H), h = (int)(u % H);
        int hkv = h / (H / Hkv);
        int hi = (H_idx == H) ? h : hkv;
        const int32_t *G = idx + ((int64_t)s * H_idx + hi) * n_idx;
        int nG = idx_len ? idx_len[(int64_t)s * H_idx + hi] : n_idx;
        row_attention(kind, Q, u * d, K, V, ((int64_t)s * Hkv + hkv) * L * d, d, scale,
                      G, nG, NULL, 0, O + u * d, lse + u);
    }
}

/* ---- dynamic top-K selection for decode queries ----
 * For query (s, h) over the keys j < len_s of its K/V head (len_s = lengths[s],
 * or L): relevance s_j = scale * q . k_j in double; G = the k = min(top_k, len_s)
 * keys with the largest s_j, equal scores ordered by the smaller j; written to
 * idx_out[s][h][0..k) in ascending j, k to len_out[s][h].  kth_out[s][h] = the
 * smallest selected score and next_out[s][h] = the largest unselected score
 * (NAN when there is none), so a caller can tell how close the cut was. */
typedef struct { double s; int32_t j; } ora_scored_t;

static int cmp_scored_desc(const void *a, const void *b)
{
    const ora_scored_t *x = (const ora_scored_t *)a, *y = (const ora_scored_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

static int cmp_i32(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

void ora_topk_select(int kind, int S, int H, int Hkv, int L, int d, double scale,
                     const void *Q, const void *K, const int32_t *lengths, int top_k,
                     int32_t *idx_out, int32_t *len_out, double *kth_out, double *next_out,
                     int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < (int64_t)S * H; ++u) {
        int s = (int)(u / H), h = (int)(u % H);
        int hkv = h / (H / Hkv);
        int len = lengths ? lengths[s] : L;
        if (len < 0) len = 0;
        if (len > L) len = L;
        int k = top_k < len ? top_k : len;
        int64_t kv_off = ((int64_t)s * Hkv + hkv) * L * d;
        ora_scored_t *sc = (ora_scored_t *)malloc(sizeof(ora_scored_t) * (size_t)(len > 0 ? len : 1));
        for (int j = 0; j < len; ++j) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += ld(Q, u * d + c, kind) * ld(K, kv_off + (int64_t)j * d + c, kind);
            sc[j].s = scale * acc;
            sc[j].j = j;
        }
        qsort(sc, (size_t)len, sizeof(ora_scored_t), cmp_scored_desc);
        int32_t *out = idx_out + u * top_k;
        for (int t = 0; t < k; ++t) out[t] = sc[t].j;
        qsort(out, (size_t)k, sizeof(int32_t), cmp_i32);
        len_out[u] = k;
        kth_out[u] = k > 0 ? sc[k - 1].s : NAN;
        next_out[u] = k < len ? sc[k].s : NAN;
        free(sc);
    }
}
