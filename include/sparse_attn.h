/*
 * sparse_attn.h -- C ABI of the B200 (sm_100a) block-sparse attention library.
 *
 * The operation (web pages on sparse attention):
 *   "Sparse Attention Weights Assumption" (1cademy), sparse attention output
 *   formula:  out_i = sum_{j in G_i} alpha'_{i,j} v_j,  G_i subset of {0..i}
 *   (causal).  alpha' is the softmax of the scaled logits s_ij = scale*q_i.k_j
 *   taken over G_i only, so a full G_i gives the glossary's dense
 *   softmax(Q K^T / sqrt(d_k)) V ("sparse attention mechanism" glossary,
 *   chipfoundryservices, "Standard Attention Bottleneck").
 *
 * G_i comes from one of four places:
 *   - sparse_attn_prefill*: a static pattern (sa_pattern_t) -- the union, by
 *     logical OR ("SAS: Sparse Attention Synthesizer", kindchill, Step 5,
 *     component 2), of a sliding window, global tokens, block-local blocks and
 *     BigBird-style random blocks (glossary, "Sparse Attention Patterns" table
 *     and "Mistral/Mixtral Sliding Window Attention"), intersected with the
 *     causal constraint -- optionally pruned by the dynamic Block-Sparse-
 *     FlashAttention rule ("Block Sparse Flash Attention", montaan AI Radio,
 *     paper summary and improvements): the exact QK^T tile of a 64-key block is
 *     computed, its maximum scaled logit is compared with a per-head calibrated
 *     threshold, and below it the block's V load and PV product are skipped and
 *     its keys leave G_i for every row of the 128-row query tile.
 *   - sparse_attn_gather: explicit index sets over a KV cache (decode).
 *   - sparse_attn_decode_window: the decode row of a causal window + global
 *     tokens pattern, over a cache of window + globals slots.
 *   - sparse_attn_decode_topk: each decode query's top_k keys by relevance
 *     score (a dynamic pattern, computed from the data at run time).
 *
 * K/V heads are shared by contiguous groups of query heads (GQA/MQA, glossary
 * "Multi-Query and Grouped-Query Attention"): h_kv = h / (H / H_kv).
 *
 * Conventions for every call below.
 *   - Tensors are caller-owned, device-resident, contiguous row-major bf16
 *     (raw IEEE bfloat16 bit patterns, passed as void*), 16-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronise, except where a comment says so.
 *   - Return value: SA_OK or an SA_ERR_* code; sparse_attn_last_error() then
 *     gives a message (thread-local).  Argument errors are detected on the host
 *     before anything is launched.
 *   - Errors found by a kernel while it runs (an index out of range in a
 *     gather set, a pipeline wait that ran out of time) are recorded in a
 *     device error word instead of faulting; read and clear it with
 *     sparse_attn_check_device_error().
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so the header needs no CUDA headers. */
typedef struct CUstream_st *sa_stream_t;

enum {
    SA_OK = 0,
    SA_ERR_INVALID_ARG = 1,   /* bad pointer, shape, alignment or descriptor           */
    SA_ERR_UNSUPPORTED = 2,   /* valid request the library has no kernel for          */
    SA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed                      */
    SA_ERR_NO_MEMORY = 4,     /* host or device allocation failed                      */
    SA_ERR_TIMEOUT = 5,       /* device: a pipeline wait ran out of time; kernel bailed */
    SA_ERR_DEVICE_INDEX = 6   /* device: a gather index was outside [0, L); row skipped */
};

/*
 * Static pattern descriptor.  G_i = { j < N : base(i, j) and (!causal or j <= i) }
 * where base is the logical OR of the primitives that are on (all keys when
 * none is on):
 *   window       W > 0.  causal: j in [i-W+1, i]  (Mistral rule, glossary);
 *                non-causal: |i - j| <= W/2 ("w nearest neighbours").
 *   n_global     g > 0.  i < g or j < g: tokens 0..g-1 see every key and are
 *                seen by every query (1cademy "Global Tokens in Attention").
 *   block_local  b > 0.  i / b == j / b (glossary "Blockwise").
 *   random       n_random > 0 and random_table != NULL: key j is visible from
 *                query i when j / random_block is listed in
 *                random_table[h][i / random_block][0 .. n_random) (BigBird).
 *   dilation     k > 1 makes the window dilated/strided (glossary "Sparse
 *                Attention Patterns": attend to every k-th token, O(N*w)):
 *                W taps k apart, i.e. (i - j) mod k == 0 and, with
 *                m = (i - j) / k, 0 <= m < W (causal) or |m| <= W/2.  The kernels
 *                run it as k independent sliding-window attentions, one per
 *                residue class i mod k, read through a strided TMA view, so no
 *                masked-out pair is computed.  Needs window > 0, no other
 *                primitive, no block-skip thresholds and N % k == 0
 *                (SA_ERR_UNSUPPORTED otherwise).  0 and 1 mean contiguous.
 * block_q x block_k is the tile of the block-skip rule and of the block FLOP
 * accounting.  The kernels tile 128 query rows x 64 keys, so block_k must be 64
 * and block_q 64 or 128 (128 when the block-skip rule is used).
 * scale: logit scale; 0 means 1/sqrt(d).
 */
typedef struct {
    int32_t causal;
    int32_t window;
    int32_t n_global;
    int32_t block_local;
    int32_t block_q;
    int32_t block_k;
    int32_t random_block;          /* multiple of 64 when random blocks are on            */
    int32_t n_random;
    const int32_t *random_table;   /* HOST pointer, int32 [H][ceil(N/random_block)][n_random],
                                      entries in [0, ceil(N/random_block)); read only while
                                      a plan is created (the plan keeps a device copy)    */
    const float *thresholds;       /* DEVICE pointer, float [H] block-skip thresholds in
                                      scaled-logit (natural-log) units, or NULL = rule off.
                                      Used by sparse_attn_prefill only; plans take the
                                      thresholds per call.                                */
    float scale;
    int32_t dilation;              /* window taps k apart; 0 or 1 = contiguous window    */
    int32_t skipped_in_denominator;/* block-skip rule variant: 1 keeps the keys of a
                                      skipped block in the softmax denominator (no V
                                      load and no PV for it, but its exp terms enter
                                      l and the running max); 0 = they leave G_i.
                                      Single-head kernel only.                          */
    int32_t row_level_skip;        /* block-skip rule, per-query reading ("Block Sparse
                                      Flash Attention", paper summary: each query's
                                      scores decide which value blocks matter): 1 = on
                                      top of the tile decision, each row drops a full
                                      block of its tile whose maximum over that row's
                                      own scaled logits is below the threshold (its
                                      keys leave that row's G_i).  The V load and PV are
                                      skipped when every row drops the block, which is
                                      the tile rule's decision.  0 = tile rule only.
                                      Not combined with skipped_in_denominator;
                                      single-head kernel only.                          */
} sa_pattern_t;

/* A compiled pattern: per-(head, 128-row query tile) lists of 64-key blocks
 * with a full/partial flag, a longest-first work order and a device copy of the
 * random table.  Owns device memory; freed by sparse_attn_plan_destroy. */
typedef struct sa_plan sa_plan_t;

typedef struct {
    int32_t T_q;            /* 128-row query tiles per (b, h): ceil(N/128); with
                               dilation k > 1, per (b, h, residue): ceil(N/k/128)       */
    int32_t n_kb;           /* 64-key blocks per row: ceil(N/64) (ceil(N/k/64))          */
    int64_t n_units;        /* work units B*H*T_q (B*k*H*T_q with dilation k > 1)        */
    int64_t blocks;         /* listed (tile, key block) pairs over all (b, h), 128x64   */
    int64_t blocks_full;    /* ... of which every pair is in G (may be skipped)         */
    int64_t blocks_desc;    /* listed blocks at the descriptor's block_q x block_k      */
    int64_t pairs;          /* sum over (b, h, i) of |G_i| of the static pattern        */
    double compile_ms;      /* host time spent compiling the pattern                    */
    int64_t split_tiles;    /* tiles whose block list is cut into pieces (see
                               sa_plan_options_t.max_unit_blocks)                       */
    int64_t queue_units;    /* entries of the work queue: whole tiles plus pieces       */
    int64_t workspace_bytes;/* device workspace of the pieces' partial results          */
} sa_plan_info_t;

/* Kernel choice for sparse_attn_plan_create_ex. */
enum {
    SA_KERNEL_AUTO = 0,          /* the kernel measured fastest for the plan's shape on
                                    B200: the single-head kernel                         */
    SA_KERNEL_SINGLE_HEAD = 1    /* the single-head kernel                                */
};

/* Compile `pat` for Q [B][H][N][d], K/V [B][H_kv][N][d].  Host work plus
 * cudaMalloc/cudaMemcpy on the current device; synchronous.  Errors:
 * SA_ERR_INVALID_ARG (shapes, H % H_kv != 0, bad descriptor or table entry),
 * SA_ERR_UNSUPPORTED (d not 64/128, block_k != 64, random_block % 64 != 0,
 * dilation k > 1 with another primitive or N % k != 0), SA_ERR_NO_MEMORY,
 * SA_ERR_CUDA.  On success *out owns the plan.  A dilated plan (k > 1) holds
 * the lists of the contiguous window over one residue class (N/k positions),
 * shared by the k classes. */
int sparse_attn_plan_create(const sa_pattern_t *pat, int B, int H, int H_kv, int N, int d,
                            sa_plan_t **out);
/* Same as sparse_attn_plan_create with an explicit kernel choice (SA_KERNEL_*;
 * other values: SA_ERR_INVALID_ARG). */
int sparse_attn_plan_create_ex(const sa_pattern_t *pat, int B, int H, int H_kv, int N, int d,
                               int kernel, sa_plan_t **out);

/* Plan options (sparse_attn_plan_create_opts).
 *
 * Split tiles: a query tile whose block list is far longer than the others
 * (the rows of global tokens attend to every key) would run on one CTA while
 * the other tiles of its head have long finished, and would read that head's
 * K and V from HBM a second time.  Such a list is cut into pieces of
 * consecutive blocks; each piece is a work unit of its own, queued with the
 * tiles of the K/V group before its own, that writes an unnormalised partial
 * result (O in fp32, the row maximum and the row sum) to a device workspace
 * owned by the plan.  Inside the same launch, the CTA that finishes the last
 * piece of a tile (a device-wide counter per tile) combines the pieces (the
 * same online-softmax combination the kernel applies across blocks) and writes
 * O and the log-sum-exp; the counters are back at zero when the launch ends.
 * Statistics, decisions and block masks are per block and do not depend on the
 * split. */
typedef struct {
    int32_t kernel;           /* SA_KERNEL_*                                             */
    int32_t max_unit_blocks;  /* 0: automatic -- a tile whose list is longer than one
                                 CTA's share of the whole launch (it alone would set
                                 the launch time) and than 2P blocks is cut into
                                 pieces of about P = max(32, 2 x the median list
                                 length) blocks, within a 256 MiB workspace; > 0:
                                 every list longer than this many blocks is cut into
                                 pieces of at most this many; < 0: no tile is split   */
} sa_plan_options_t;

/* Same as sparse_attn_plan_create with options (NULL: kernel SA_KERNEL_AUTO,
 * max_unit_blocks 0).  Errors as sparse_attn_plan_create; SA_ERR_INVALID_ARG
 * for an unknown kernel value. */
int sparse_attn_plan_create_opts(const sa_pattern_t *pat, int B, int H, int H_kv, int N, int d,
                                 const sa_plan_options_t *opts, sa_plan_t **out);
int sparse_attn_plan_info(const sa_plan_t *plan, sa_plan_info_t *info);
void sparse_attn_plan_destroy(sa_plan_t *plan);   /* synchronises the device; NULL ok */

/* Prefill with a compiled plan.
 *   Q [B][H][N][d], K, V [B][H_kv][N][d] (bf16, device, read); O [B][H][N][d]
 *   (bf16, device, written).
 *   thresholds: device float [H] (block-skip rule on) or NULL (static pattern only).
 *   lse_out: device float [B][H][N] = ln sum_{j in G_i} exp(s_ij), -inf for an
 *            empty G_i; or NULL.
 *   block_mask_out: device uint8 [B][H][T_q][n_kb]; 0 = block not listed,
 *            1 = computed and kept, 2 = skipped by the rule; or NULL.
 *   block_stat_out: device float [B][H][T_q][n_kb]; for listed blocks the
 *            maximum scaled logit over the tile's visible pairs (unlisted
 *            entries are left untouched); or NULL.
 * A dilated plan takes no thresholds, block_mask_out or block_stat_out
 * (SA_ERR_UNSUPPORTED): the block-skip rule is defined on contiguous tiles.
 * The plan must not be destroyed while a launch that uses it may still run,
 * and launches that use one plan must not overlap on the GPU (issue them on
 * one stream, or order them): the plan holds the launch's work-queue
 * counters. */
int sparse_attn_prefill_plan(const sa_plan_t *plan, const void *Q, const void *K,
                             const void *V, void *O, const float *thresholds,
                             float *lse_out, uint8_t *block_mask_out,
                             float *block_stat_out, sa_stream_t stream);

/* One-shot prefill: looks the pattern up in a per-process plan cache (keyed on
 * every descriptor field, the random table's contents and the shapes), compiles
 * it on a miss (synchronous, see sparse_attn_plan_create), then launches as
 * sparse_attn_prefill_plan with pat->thresholds.  Calls that hit the same
 * cached plan share its work-queue counters, so they must not overlap on the
 * GPU either (one stream, or ordered streams). */
int sparse_attn_prefill(const void *Q, const void *K, const void *V, void *O,
                        int B, int H, int H_kv, int N, int d, const sa_pattern_t *pat,
                        float *lse_out, uint8_t *block_mask_out, sa_stream_t stream);

/* Block-statistics pass of the block-skip rule over a plan: computes the
 * QK^T tiles of every listed block and writes block_stat_out (layout as
 * above) and block_mask_out (1 for every listed block); no V is read and no
 * output is written.  Used to calibrate thresholds on a calibration draw.
 * Dilated plans: SA_ERR_UNSUPPORTED. */
int sparse_attn_block_stats(const sa_plan_t *plan, const void *Q, const void *K,
                            float *block_stat_out, uint8_t *block_mask_out,
                            sa_stream_t stream);

/* Per-head threshold calibration from a statistics pass: for each head h,
 * thresholds_out[h] = the element of rank floor((n_h - 1) * q) (0-based,
 * ascending) among the statistics of head h's FULL blocks over all b and
 * tiles, n_h their number (q = 0.5 gives the lower median).  block_stat is
 * the output of sparse_attn_block_stats for the same plan.  Device float [H]
 * out; -inf when a head has no full block. */
int sparse_attn_calibrate(const sa_plan_t *plan, const float *block_stat, double q,
                          float *thresholds_out, sa_stream_t stream);

/* Explicit index-set attention over a KV cache (decode, one query per sequence).
 *   Q [S][H][d] bf16; K, V [S][H_kv][L][d] bf16; O [S][H][d] bf16 (written).
 *   idx: device int32 [S][H_idx][n_idx]; each set unique, in [0, L); rows are
 *        visited in the order given (the workloads pass them sorted ascending;
 *        the order changes only the rounding).  H_idx == H: one set per query
 *        head; H_idx == H_kv: one set per K/V head, shared by its query heads.
 *   idx_len: device int32 [S][H_idx] (entries used, 0..n_idx) or NULL (= n_idx).
 *   lse_out: device float [S][H] or NULL.
 *   An empty set gives O = 0, lse = -inf.  An index outside [0, L) is skipped
 *   and recorded as SA_ERR_DEVICE_INDEX in the device error word. */
int sparse_attn_gather(const void *Q, const void *K, const void *V, const int32_t *idx,
                       const int32_t *idx_len, void *O, int S, int H, int H_kv, int H_idx,
                       int L, int n_idx, int d, float scale, float *lse_out,
                       sa_stream_t stream);

/* Decode over a minimum-size KV cache for the causal pattern "sliding window
 * of W keys OR the first g (global) tokens" (glossary, "Mistral/Mixtral
 * Sliding Window Attention" and "Sparse Attention Patterns"; the cache that
 * the SAS tutorial's geometric pattern analyzer sizes from the pattern, Step 5,
 * component 3).  The query of sequence s sits at position p = positions[s]; its
 * index set is G_p = [0, min(g, p+1)) u [max(g, p-W+1), p], derived on the
 * device from the descriptor -- no index array.
 *   pat: causal = 1, window = W >= 1, n_global = g >= 0; no block_local, no
 *        random blocks, no thresholds (otherwise SA_ERR_UNSUPPORTED); scale as
 *        in sa_pattern_t.
 *   Cache: K, V [S][H_kv][C][d] bf16 with C = W + g slots per (sequence, K/V
 *        head): key j lives in slot sparse_attn_window_slot(j, W, g) (j for
 *        j < g, else g + (j mod W)); the caller writes keys 0..p in order, so
 *        the ring slots hold the last W keys.
 *   Q [S][H][d] bf16, O [S][H][d] bf16 (written), positions device int32 [S],
 *   lse_out device float [S][H] or NULL.  Rows are visited in ascending key
 *   order, so the result equals sparse_attn_gather over the same cache with
 *   the slots of G_p as the index set.  A negative position is recorded as
 *   SA_ERR_DEVICE_INDEX and gives O = 0, lse = -inf. */
int sparse_attn_decode_window(const void *Q, const void *K, const void *V,
                              const int32_t *positions, void *O, int S, int H, int H_kv,
                              int d, const sa_pattern_t *pat, float *lse_out,
                              sa_stream_t stream);

/* Decode attention over the top_k keys of each query: the dynamic primitive
 * "attend to the top-K dynamic tokens" ("SAS: Sparse Attention Synthesizer",
 * Step 5, component 1, primitive C; the dynamic sparse patterns of "Sparse
 * Attention Weights Assumption", whose G holds the tokens with the highest
 * relevance scores).  For query (s, h) over the keys j < len_s of its K/V head:
 * relevance s_j = scale * q . k_j (fp32), G = the k = min(top_k, len_s) keys
 * with the largest s_j, equal scores to the smaller j; out = sum over G of
 * softmax_G(s_j) v_j, lse = ln sum_G exp(s_j) (-inf and O = 0 for len_s = 0).
 *   Q [S][H][d], K, V [S][H_kv][L][d] (bf16, device, read); O [S][H][d] (written).
 *   lengths: device int32 [S] keys per sequence in [0, L], or NULL (all L);
 *            a length outside [0, L] is clamped and recorded as SA_ERR_DEVICE_INDEX.
 *   idx_out: device int32 [S][H][top_k] or NULL: the selected keys, ascending,
 *            in the first idx_len entries (the rest untouched);
 *   idx_len_out: device int32 [S][H] or NULL: k per query.
 *   lse_out: device float [S][H] or NULL.
 *   workspace: device memory of sparse_attn_decode_topk_workspace(S, H, L,
 *            top_k) bytes, 16-byte aligned, owned by the caller, not read before
 *            it is written; calls that overlap on the GPU need separate ones.
 *   scale: 0 means 1/sqrt(d).
 * Three kernels on `stream` (a score pass that reads every K row once per K/V
 * head, an exact radix select that also writes the selected keys' scores, an
 * attention pass over the selected V rows and those scores) plus a memset of
 * the workspace histogram.  Errors: SA_ERR_INVALID_ARG
 * (shapes, H % H_kv, top_k < 1, alignment, workspace too small),
 * SA_ERR_UNSUPPORTED (d not 64/128, sizes past 32-bit grid limits). */
size_t sparse_attn_decode_topk_workspace(int S, int H, int L, int top_k);
int sparse_attn_decode_topk(const void *Q, const void *K, const void *V, const int32_t *lengths,
                            void *O, int S, int H, int H_kv, int L, int d, int top_k,
                            float scale, int32_t *idx_out, int32_t *idx_len_out,
                            float *lse_out, void *workspace, size_t workspace_bytes,
                            sa_stream_t stream);

/* Cache slot of key j (j >= 0) in the layout of sparse_attn_decode_window;
 * -1 when j < 0, window < 1 or n_global < 0.  Host only. */
int64_t sparse_attn_window_slot(int64_t j, int window, int n_global);

/* Prefill that allocates no device memory.  (The pages have no counterpart:
 * this is a deployment variant of sparse_attn_prefill.)  For callers that
 * cannot call cudaMalloc at run time -- code whose device memory is owned by
 * an external pool or allocator, or runtimes that forbid allocation on the
 * inference path.  Same arguments and result as sparse_attn_prefill (block
 * mask output excepted); the compiled pattern is not cached but rebuilt on the
 * host each call and copied into a fixed 8 MiB static device array.  CUDA
 * loads the library's device code lazily, so the array is reserved on a
 * device when that code is first used there (for a caller of this entry point
 * alone: its first call) and held until the process exits; make a warm-up call
 * before an external pool takes the rest of the device.  Patterns whose block
 * lists, work order and random table need more than 8 MiB are rejected with
 * SA_ERR_INVALID_ARG; every check runs on the host before the first CUDA call,
 * so a rejected call queues no device work.  The first call on a device looks up the array's
 * device address (with that device current); make it before any stream
 * capture.  Every call reuses the array: calls that can overlap on the GPU
 * (different streams without ordering) race; calls on one stream do not.
 * No tile is split into pieces here (the pieces' workspace would not fit the
 * array): every tile is one work unit, as with max_unit_blocks < 0.
 * Calls no cudaMalloc, cudaFree or other allocating library routine. */
int sparse_attn_prefill_noalloc(const void *Q, const void *K, const void *V, void *O,
                                int B, int H, int H_kv, int N, int d, const sa_pattern_t *pat,
                                float *lse_out, sa_stream_t stream);

/* Host-only work order (no GPU needed): the prefill queue a plan built with
 * these arguments and options->max_unit_blocks holds.  First call with
 * units == NULL to get *n_units_out (queue entries), *n_pieces_out and
 * *n_split_out; then again with units int32 [n_units], pieces int32
 * [n_pieces][4] and split int32 [n_split][4].  units[k] >= 0 is a whole tile
 * ((b'*H + h)*T + t, b' = b*k + residue with dilation k); units[k] < 0 is
 * piece ~units[k] = {tile, first block of the list, blocks, workspace slot};
 * split[s] = {tile, first slot, pieces, 0}.  Errors as sparse_attn_plan_create
 * (no SA_ERR_CUDA / SA_ERR_NO_MEMORY). */
int sparse_attn_work_order(const sa_pattern_t *pat, int B, int H, int H_kv, int N, int d,
                           int max_unit_blocks, int64_t *n_units_out, int64_t *n_pieces_out,
                           int64_t *n_split_out, int32_t *units, int32_t *pieces,
                           int32_t *split);

/* Host-only pattern compiler (no GPU needed): the block lists a plan holds, at
 * tile_q x tile_k granularity.  H_pat = H when random blocks are on, else 1
 * (the lists do not depend on the head).  First call with row_ptr == NULL to
 * get *H_pat_out, *T_out, *n_entries_out; then call again with
 * row_ptr int32 [H_pat*T + 1], kb int32 [n_entries], full uint8 [n_entries]
 * and, optionally, cnt int64 [n_entries] (visible pairs per listed block).
 * With dilation k > 1 the lists are those of one residue class: the
 * contiguous window over N/k positions (T = ceil(N/k/tile_q)). */
int sparse_attn_compile_pattern(const sa_pattern_t *pat, int H, int N, int tile_q,
                                int tile_k, int *H_pat_out, int *T_out,
                                int64_t *n_entries_out, int32_t *row_ptr, int32_t *kb,
                                uint8_t *full, int64_t *cnt);

/* Waits for `stream`, then reads and clears the device error word.  Returns
 * SA_OK, SA_ERR_TIMEOUT, SA_ERR_DEVICE_INDEX or SA_ERR_CUDA. */
int sparse_attn_check_device_error(sa_stream_t stream);

/* Message for the last error on this thread ("" if none). */
const char *sparse_attn_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* SPARSE_ATTN_H */
