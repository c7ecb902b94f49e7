/*
 * qsa.h -- C ABI of libqsa.so: Qwen Sparse Attention (QSA) on NVIDIA B200 (sm_100a).
 *
 * QSA replaces a full-attention layer by micro-block sparse softmax attention
 * with a compressed lightweight indexer.  Source for every operation below:
 * "On the Design of Qwen3.8 Next Architecture: Evaluation, Efficiency, and
 * Training Stability" (reading notes), section 6 "GDN 连续压缩与 QSA 精确检索"
 * (pooled-key equation, indexer equation, budget sentence, complexity
 * equation) and its "Model Summary" table (head counts and sizes).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor pointer is DEVICE memory owned by the caller; the library
 *    never allocates, frees or keeps a pointer after the call returns.  Host
 *    arguments are plain integers/floats and the config struct (read during
 *    the call only).
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream) and launch on the current device.
 *  - Return value: QSA_OK when the work was enqueued; QSA_ERR_INVALID_ARG /
 *    QSA_ERR_UNSUPPORTED / QSA_ERR_WORKSPACE_TOO_SMALL are detected on the
 *    host BEFORE anything is launched; QSA_ERR_CUDA reports a launch error.
 *    Errors found on the device (an index out of range, a bounded wait that
 *    gave up) do not abort the launch: the kernel records QSA_ERR_DEVICE_CHECK
 *    or QSA_ERR_TIMEOUT in a sticky per-device status word and skips the
 *    offending work; read it with qsa_get_device_status().
 *  - bf16 tensors are raw 16-bit patterns (qsa_bf16).  Layouts are dense,
 *    row-major, innermost dimension last, no padding.
 *  - Variable-length batches are packed.  cu_seqlens_q / cu_seqlens_k /
 *    cu_blocks are int32 device arrays of batch+1 prefix sums (first entry 0)
 *    of L_q,s, L_k,s and floor(L_k,s / r).  Query row i of sequence s sits at
 *    position t = (L_k,s - L_q,s) + (i - cu_seqlens_q[s]) (bottom-right
 *    aligned: prefill has L_q = L_k, decode has L_q = 1).
 *  - Notation: r = micro-block size, b_t = floor(t / r) is the query's own
 *    block, the candidates of t are the complete blocks 0 .. b_t - 1, and
 *    k = budget_blocks counts the own block (|Sel_t| = min(k, b_t + 1)).
 *  - Supported configuration: the model's (r = 4, 24 query heads, 2 KV
 *    heads, head dim 256, 4 indexer heads of dim 128) with a budget of
 *    k <= 2048 blocks (the model uses 512); anything else returns
 *    QSA_ERR_UNSUPPORTED.
 *  - Thread safety: calls may come from several host threads.  Host-side
 *    state is set up once and guarded by locks: the driver's tensor-map
 *    encoder, each kernel's shared-memory opt-in (once per device) and the
 *    static-scratch address (once per device).  The device keeps one sticky
 *    status word per device.  Work on the GPU is ordered by the caller's
 *    streams; only qsa_sparse_attn_decode_static_scratch shares memory
 *    between calls (see there).
 */
#ifndef QSA_H
#define QSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t qsa_status;
#define QSA_OK 0
#define QSA_ERR_INVALID_ARG 1
#define QSA_ERR_UNSUPPORTED 2
#define QSA_ERR_WORKSPACE_TOO_SMALL 3
#define QSA_ERR_CUDA 4
#define QSA_ERR_TIMEOUT 5
#define QSA_ERR_DEVICE_CHECK 6
#define QSA_ERR_SCRATCH_LIMIT 7 /* the call needs more than QSA_STATIC_SCRATCH_BYTES */

typedef uint16_t qsa_bf16; /* bfloat16 bit pattern */

/* flags */
#define QSA_COMPRESS_NO_NORM 0x1u /* plain mean-pool, no RMSNorm in the compressor */
#define QSA_INDEX_ROPE 0x2u       /* partial RoPE of the pooled indexer key (rope_dims, rope_base) */

typedef struct qsa_config {
    int32_t r;             /* micro-block size (4) */
    int32_t budget_blocks; /* k: blocks kept per query, own block included (512) */
    int32_t n_heads_q;     /* 24 */
    int32_t n_heads_kv;    /* 2 (GQA: head h reads KV group h / 12) */
    int32_t head_dim;      /* 256 */
    int32_t n_heads_idx;   /* indexer query heads (4); one shared key head */
    int32_t idx_dim;       /* indexer head dim (128) */
    float softmax_scale;   /* 1/sqrt(256) */
    float rms_eps;         /* compressor RMSNorm eps (1e-6) */
    uint32_t flags;        /* QSA_COMPRESS_NO_NORM | QSA_INDEX_ROPE */
    int32_t kv_chunk_blocks; /* > 0: key-chunk size (micro-blocks) of the L2-blocked prefill
                                schedule; 0 (default): one pass per query */
    int32_t rope_dims;     /* with QSA_INDEX_ROPE: rotated leading dims of the indexer head
                              (a multiple of 8, at most idx_dim; default 64) */
    float rope_base;       /* with QSA_INDEX_ROPE: frequency base (default 10000) */
} qsa_config;

/* op ids for qsa_workspace_size */
#define QSA_OP_COMPRESS 0
#define QSA_OP_INDEX 1
#define QSA_OP_SELECT 2
#define QSA_OP_PREFILL 3
#define QSA_OP_DECODE 4
#define QSA_OP_DENSE 5
#define QSA_OP_DECODE_PAGED 6 /* qsa_sparse_attn_decode_paged */
#define QSA_OP_INDEX_SELECT 7 /* qsa_index_select */
#define QSA_OP_INDEX_SELECT_PAGED 8 /* qsa_index_select_paged */
#define QSA_OP_DECODE_MTP 9 /* qsa_sparse_attn_decode_mtp */

/* Fill *cfg with the model's values (r 4, k 512, 24/2/256, 4/128, scale 1/16,
 * eps 1e-6, flags 0, kv_chunk_blocks 0, rope_dims 64, rope_base 10000).  Host only. */
void qsa_config_init(qsa_config *cfg);

/*
 * Key compressor -- pooled-key equation of section 6:
 *   kc[b] = RMSNorm( (1/r) * sum_{j<r} k_idx[b r + j] ),   unit gain, eps cfg->rms_eps
 * for every complete block b < floor(L_k,s / r) of every sequence (the mean
 * alone with QSA_COMPRESS_NO_NORM).  fp32 arithmetic.  Each value x is stored as
 * a compensated bf16 pair, hi = bf16(x) and lo = bf16(x - hi) (round to nearest
 * even), so kc = hi + lo carries about 16 significant bits: a single 16-bit
 * value (bf16, and in rows of small scores fp16 too) shifts indexer scores by
 * more than the selection tolerance.
 *   k_idx      [total_k, idx_dim] bf16   raw indexer keys (one shared key head)
 *   cu_seqlens_k, cu_blocks  [batch+1] int32
 *   total_k    host: rows of k_idx (bounds the launch)
 *   blk_begin  [batch] int32 or NULL.  NULL: every complete block is written.
 *              Otherwise only blocks [blk_begin[s], blk_begin[s] + max_new_blocks)
 *              that are complete (a decode step refreshes the blocks it completed).
 *   kc         [cu_blocks[batch], 2, idx_dim] bf16, written: per block the hi
 *              plane, then the lo plane.
 * QSA_INDEX_ROPE (the sentence before the pooled-key equation: pool first, then a
 * partial RoPE, so keys of different rotation phases are never averaged; the
 * pages fix no dims, base or position): after the pool and the norm, the first
 * cfg->rope_dims dims rotate in pairs (i, i + rope_dims/2) by the angle
 * (b r) * rope_base^(-2i / rope_dims), b r the block's first position; angles and
 * their sines in fp64.  The indexer queries must then be rotated at their own
 * positions t (qsa_rope_queries), as the attention's q and k arrive rotated.
 */
qsa_status qsa_compress_keys(const qsa_config *cfg, const qsa_bf16 *k_idx,
                             const int32_t *cu_seqlens_k, const int32_t *cu_blocks,
                             int32_t batch, int64_t total_k, const int32_t *blk_begin,
                             int32_t max_new_blocks, qsa_bf16 *kc, void *stream);

/*
 * Partial RoPE of the indexer queries, in place: row i of sequence s sits at
 * t = (L_k,s - L_q,s) + (i - cu_seqlens_q[s]) and every head of it rotates as the
 * pooled keys do under QSA_INDEX_ROPE (same dims, pairs and base; angle t * f_i).
 * fp32 arithmetic on the bf16 values, fp64 angles, bf16 round-to-nearest-even
 * stores.  Requires QSA_INDEX_ROPE in cfg->flags (QSA_ERR_INVALID_ARG otherwise).
 *   q_idx      [total_q, n_heads_idx, idx_dim] bf16, read and written
 *   cu_seqlens_q, cu_seqlens_k  [batch+1] int32
 *   total_q    host: rows of q_idx
 */
qsa_status qsa_rope_queries(const qsa_config *cfg, qsa_bf16 *q_idx, const int32_t *cu_seqlens_q,
                            const int32_t *cu_seqlens_k, int32_t batch, int64_t total_q, void *stream);

/*
 * Indexer scores -- indexer equation of section 6, with one weight per
 * (query, indexer head) (w = 1 gives the equation as printed):
 *   S[t, b] = sum_h w[t, h] * max(0, <q_idx[t, h, :], kc[b, :]>),   b < b_t
 * bf16 tensor-core products (q_idx . hi + q_idx . lo), fp32 accumulation and epilogue.
 *   q_idx   [total_q, n_heads_idx, idx_dim] bf16;  w [total_q, n_heads_idx] fp32
 *   kc      [kc_rows, 2, idx_dim] bf16 hi/lo pairs (the compressor's output; kc_rows =
 *           cu_blocks[batch]); both planes enter the products
 *   rows    packed query rows [row_begin, row_end) are scored (a chunk of a prefill)
 *   scores  fp32, row i at scores + (i - row_begin) * ld; entries b < b_t(i) hold
 *           the scores, entries b_t(i) <= b < ld are left as they were.
 *           ld >= every b_t(i).
 *   total_q host: rows of q_idx; max_len_q host: max over s of L_q,s (a launch hint:
 *           1 selects the one-row-per-sequence decode kernel)
 * Workspace: none (ws may be NULL).
 */
qsa_status qsa_index_scores(const qsa_config *cfg, const qsa_bf16 *q_idx, const float *w,
                            const qsa_bf16 *kc, int64_t kc_rows,
                            const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                            const int32_t *cu_blocks, int32_t batch, int64_t total_q,
                            int32_t max_len_q, int64_t row_begin, int64_t row_end,
                            float *scores, int64_t ld, void *ws, size_t ws_bytes, void *stream);

/*
 * Top-k block selection -- budget sentence of section 6: the own block b_t is
 * always kept; the other min(k - 1, b_t) slots go to the highest-scoring
 * candidates 0 .. b_t - 1, ties to the lower block index.  Exact on the fp32
 * score bits (radix select on an order-preserving integer key; -0.0 == +0.0).
 *   scores  as written by qsa_index_scores for rows [row_begin, row_end), stride ld
 *   sel     [total_q, k] int32: row i at sel + i * k (absolute packed row), block ids
 *           local to the sequence, ascending, padded with -1.
 * NaN scores give an unspecified (but valid) selection.  Workspace: none.
 */
qsa_status qsa_select_blocks(const qsa_config *cfg, const float *scores, int64_t ld,
                             const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                             int32_t batch, int64_t row_begin, int64_t row_end, int32_t *sel,
                             void *ws, size_t ws_bytes, void *stream);

/*
 * Fused indexer + top-k selection -- the indexer equation, the budget sentence
 * and the O(n^2 / r) complexity equation of section 6: for packed rows
 * [row_begin, row_end), the same selection qsa_select_blocks makes on the scores
 * of qsa_index_scores (same arguments as those two calls), without writing the
 * rows' full score rows to memory.  Prefill rows (max_len_q > 1), per row:
 *   - the tensor-core indexer scores every stride-th 128-block kc tile into a
 *     compact sample, and a lower bound theta of the row's (k-1)-th best score is
 *     the sample's r_lo-th best, r_lo = mu + 4 sqrt(mu) + 8 (mu = the expected
 *     number of the row's winners in the sample);
 *   - the indexer scores every tile and appends (score, block) with score >= theta
 *     to the row's candidate list (4 k entries);
 *   - the exact top k - 1 of the list is the row's selection whenever the list
 *     holds at least k - 1 entries and did not overflow (every block that can win,
 *     ties included, is then in the list); otherwise the row's full score row is
 *     recomputed on CUDA cores into workspace scratch and selected from there.
 * The tensor-core scores are the same fp32 values qsa_index_scores stores, so
 * the selection equals the materialised path's bit for bit, except for rows that
 * take the fallback, whose scores carry CUDA-core fp32 rounding.
 * Decode rows (max_len_q == 1): the one-row indexer reads only the hi plane of kc
 * (half the bytes of the exact scan) into the workspace.  With the RMSNorm every
 * ||kc_b|| <= sqrt(idx_dim) and the lo plane is hi's rounding residue, so each such
 * score is within E = sum_h |w_h| ||q_h|| sqrt(idx_dim) (2^-8 1.01 + 1e-4) of the
 * exact one; the blocks within 2E of the row's (k-1)-th best are rescored exactly
 * (hi + lo) and the row's exact top k - 1 is taken among them -- the same selection
 * as qsa_index_scores + qsa_select_blocks.  A row whose candidate list exceeds 4096
 * blocks or whose sampled bound fails, and every row under QSA_COMPRESS_NO_NORM, takes
 * the exact scan of the whole row instead (same selection).
 *   max_len_k  host: an upper bound of every L_k,s (sizes the samples and scratch)
 *   sel        [total_q, k] int32 as qsa_select_blocks writes it
 * Workspace: qsa_workspace_size(cfg, QSA_OP_INDEX_SELECT, batch, row_end - row_begin,
 * max_len_k) bytes, 16-byte aligned (about 576 MB for 16384 rows at 262144 tokens,
 * against 4.3 GB of materialised scores).
 */
qsa_status qsa_index_select(const qsa_config *cfg, const qsa_bf16 *q_idx, const float *w, const qsa_bf16 *kc,
                            int64_t kc_rows, const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                            const int32_t *cu_blocks, int32_t batch, int64_t total_q, int32_t max_len_q,
                            int64_t max_len_k, int64_t row_begin, int64_t row_end, int32_t *sel, void *ws,
                            size_t ws_bytes, void *stream);

/*
 * The compressed-key side of a paged decode cache.  The reading notes' decode
 * measurement ("结果 2") compares against a paged GQA cache; here every per-token
 * tensor of a sequence lives in fixed-size pages found through ONE block table:
 *   block_table  [batch, max_pages] int32 (device): page j of sequence s holds its
 *                tokens [j page_size, (j + 1) page_size); ids in 0 .. num_pages - 1
 *   page_size    a multiple of r (a micro-block never straddles a page)
 *   k_idx_pages  [num_pages, page_size, idx_dim] bf16: raw indexer keys
 *   kc_pages     [num_pages, page_size / r, 2, idx_dim] bf16 hi/lo pairs; block b
 *                of sequence s is row (b r mod page_size) / r of page
 *                block_table[s][b r / page_size]
 * K/V pages for qsa_sparse_attn_decode_paged use the same table.  Lengths come from
 * cu_seqlens_k [batch + 1] (only L_s = cu[s+1] - cu[s] is used).  A page id out of
 * range is skipped (compress) or read as page row 0 (index) and flags
 * QSA_ERR_DEVICE_CHECK.
 *
 * qsa_compress_keys_paged: the pooled-key equation of section 6 (the same
 * arithmetic and hi/lo store as qsa_compress_keys) for every complete block of
 * every sequence (blk_begin == NULL; max_len_k bounds every L_s), or, with
 * blk_begin [batch], for blocks [blk_begin[s], blk_begin[s] + max_new_blocks) that
 * are complete (a decode step refreshes the block it completed).
 */
qsa_status qsa_compress_keys_paged(const qsa_config *cfg, const qsa_bf16 *k_idx_pages, qsa_bf16 *kc_pages,
                                   int64_t num_pages, int32_t page_size, const int32_t *block_table,
                                   int32_t max_pages, const int32_t *cu_seqlens_k, int32_t batch, int64_t max_len_k,
                                   const int32_t *blk_begin, int32_t max_new_blocks, void *stream);

/*
 * qsa_index_select_paged: decode indexer + top-k selection over a paged kc cache,
 * one new query per sequence at t = L_s - 1 (indexer equation and budget sentence
 * of section 6): the same scores (CUDA-core fp32 GEMV) and the same selection as
 * qsa_index_scores (max_len_q = 1) + qsa_select_blocks on the packed cache.
 *   q_idx [batch, n_heads_idx, idx_dim] bf16; w [batch, n_heads_idx] fp32
 *   sel   [batch, k] int32 (ascending, -1 padded)
 *   max_len_k  host: an upper bound of every L_s
 * Workspace: qsa_workspace_size(cfg, QSA_OP_INDEX_SELECT_PAGED, batch, batch,
 * max_len_k) bytes (one fp32 score row per sequence), 16-byte aligned.
 */
qsa_status qsa_index_select_paged(const qsa_config *cfg, const qsa_bf16 *q_idx, const float *w,
                                  const qsa_bf16 *kc_pages, int64_t num_pages, int32_t page_size,
                                  const int32_t *block_table, int32_t max_pages, const int32_t *cu_seqlens_k,
                                  int32_t batch, int64_t max_len_k, int32_t *sel, void *ws, size_t ws_bytes,
                                  void *stream);

/*
 * Sparse GQA attention, prefill -- expansion + core attention of section 6:
 * query t attends, per head h with KV group g = h / (n_heads_q / n_heads_kv), to
 * the tokens of its selected blocks, [b r, b r + r) cut to j <= t:
 *   o[t, h] = sum_j softmax_j(scale * <q[t, h], k[j, g]>) v[j, g]
 * bf16 tensor-core products, fp32 softmax and accumulation, bf16 output.
 *   q   [total_q, n_heads_q, head_dim] bf16; k, v [total_k, n_heads_kv, head_dim] bf16
 *   sel [total_q, k] int32 as produced by qsa_select_blocks (ascending, -1 = unused)
 *   rows [row_begin, row_end) of the packed queries are computed
 *   o   [total_q, n_heads_q, head_dim] bf16 written for those rows
 *   lse [total_q, n_heads_q] fp32 natural-log sum-exp of the scaled logits, or NULL
 *   max_len_k host: max over s of L_k,s
 * A selected block id outside 0 .. b_t is skipped and flagged QSA_ERR_DEVICE_CHECK.
 * Workspace: none by default.  With cfg->kv_chunk_blocks > 0 and
 * qsa_workspace_size(cfg, QSA_OP_PREFILL, batch, row_end - row_begin, max_len_k)
 * bytes, the rows are processed key chunk by key chunk (chunk-major, so the
 * gathers of a chunk hit L2) and the per-chunk softmax states are merged by a
 * second kernel; with less (or NULL) one pass per query is used.  Both compute
 * the same function.  (On B200 at 262144 tokens the single pass is faster: the
 * gather is bound by the per-SM pipeline, not by DRAM, and the merge costs.)
 */
qsa_status qsa_sparse_attn_prefill(const qsa_config *cfg, const qsa_bf16 *q, const qsa_bf16 *k,
                                   const qsa_bf16 *v, const int32_t *sel,
                                   const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                   int32_t batch, int64_t total_q, int64_t total_k, int64_t max_len_k,
                                   int64_t row_begin, int64_t row_end, qsa_bf16 *o, float *lse,
                                   void *ws, size_t ws_bytes, void *stream);

/*
 * Sparse GQA attention, decode: one new query per sequence at t = L_k,s - 1,
 * same definition as the prefill.  Below two sequences per SM the batch's
 * 64-token tiles are spread evenly over the CTAs, cutting sequences into
 * pieces whose partial softmax states (m, l, o) a second kernel merges; from
 * two sequences per SM on, every CTA attends whole sequences.
 *   q [batch, n_heads_q, head_dim] bf16; k_cache, v_cache [total_k, n_heads_kv,
 *   head_dim] bf16 (packed, the new token included); sel [batch, k] int32;
 *   o [batch, n_heads_q, head_dim] bf16; lse [batch, n_heads_q] fp32 or NULL.
 * Workspace: qsa_workspace_size(cfg, QSA_OP_DECODE, batch, batch, 0) bytes.
 */
qsa_status qsa_sparse_attn_decode(const qsa_config *cfg, const qsa_bf16 *q,
                                  const qsa_bf16 *k_cache, const qsa_bf16 *v_cache,
                                  const int32_t *cu_seqlens_k, int32_t batch, int64_t total_k,
                                  const int32_t *sel, qsa_bf16 *o, float *lse, void *ws,
                                  size_t ws_bytes, void *stream);

/*
 * Sparse GQA attention, decode, over a paged K/V cache: the same result as
 * qsa_sparse_attn_decode, with the K/V rows of sequence s found through its
 * block table instead of a packed cache.  Only the attention reads pages; the
 * compressed keys, the indexer and the selector keep their packed layout.
 *   k_pages, v_pages [num_pages, page_size, n_heads_kv, head_dim] bf16: the pool
 *   block_table [batch, max_pages] int32 (device): page j of sequence s holds its
 *     tokens [j page_size, (j + 1) page_size); page ids in 0 .. num_pages - 1
 *   cu_seqlens_k [batch + 1] int32 (device): only the lengths L_s = cu[s+1] - cu[s]
 *     are used here (t = L_s - 1)
 *   page_size: a multiple of r (a micro-block never straddles pages);
 *     num_pages * page_size * n_heads_kv < 2^31.
 * The batch's tiles are always spread evenly over the CTAs (pieces merged by a
 * second kernel).  Workspace: qsa_workspace_size(cfg, QSA_OP_DECODE_PAGED, batch,
 * batch, 0) bytes.  A page id out of range reads zeros and flags
 * QSA_ERR_DEVICE_CHECK.  The pages' own dense baseline uses a paged GQA cache.
 */
qsa_status qsa_sparse_attn_decode_paged(const qsa_config *cfg, const qsa_bf16 *q, const qsa_bf16 *k_pages,
                                        const qsa_bf16 *v_pages, int64_t num_pages, int32_t page_size,
                                        const int32_t *block_table, int32_t max_pages,
                                        const int32_t *cu_seqlens_k, int32_t batch, const int32_t *sel,
                                        qsa_bf16 *o, float *lse, void *ws, size_t ws_bytes, void *stream);

/*
 * Context-parallel decode, one shard: a long-context decode whose K/V cache is split
 * by block ranges over GPUs, one process per GPU.  The shard holds, for every
 * sequence s, the global micro-blocks [blk_lo[s], blk_hi[s]) of its cache, whose
 * tokens sit in k_local / v_local from row tok_local[s] on (the shard that holds a
 * sequence's last block also holds its partial tail, up to L_s).  Every shard gets
 * the same selection (qsa_select_blocks over the shards' score rows, see below) and
 * attends only its own selected blocks: an id outside its window is skipped without
 * a flag (another shard holds it); ids outside 0 .. b_t are flagged as always.
 * o and lse are the shard's partial state: softmax over its blocks only (a row with
 * none gets o = 0, lse = -inf).  qsa_merge_attn_states then gives the result of
 * qsa_sparse_attn_decode over the whole cache (up to rounding).
 *   cu_seqlens_k  [batch+1] int32: the sequences' GLOBAL lengths (t = L_s - 1)
 *   tok_local     [batch] int64; blk_lo, blk_hi [batch] int32 (device)
 *   k_local, v_local [total_k_local, n_heads_kv, head_dim] bf16
 *   lse           [batch, n_heads_q] fp32 (required)
 * The even schedule only (batch < 2 x the CTAs of the GPU, else QSA_ERR_UNSUPPORTED).
 * Workspace: qsa_workspace_size(cfg, QSA_OP_DECODE_PAGED, batch, batch, 0) bytes.
 *
 * The shards' indexer scores: each shard scores its own blocks (qsa_index_scores
 * with its compressed keys and per-sequence lengths L' with floor((L' - 1) / r) = n,
 * its candidate blocks, and floor(L' / r) = its complete blocks) into its columns of
 * a [batch, ld] row buffer; a sum over the shards
 * (NCCL all-reduce; disjoint columns) gives every shard the full rows, and
 * qsa_select_blocks on them gives the one-GPU selection bit for bit.
 */
qsa_status qsa_sparse_attn_decode_window(const qsa_config *cfg, const qsa_bf16 *q, const qsa_bf16 *k_local,
                                         const qsa_bf16 *v_local, const int32_t *cu_seqlens_k, int32_t batch,
                                         int64_t total_k_local, const int64_t *tok_local, const int32_t *blk_lo,
                                         const int32_t *blk_hi, const int32_t *sel, qsa_bf16 *o, float *lse,
                                         void *ws, size_t ws_bytes, void *stream);

/*
 * Merge of partial attention states of the same rows (context-parallel shards):
 *   lse = log sum_p exp(lse_p),  o = sum_p exp(lse_p - lse) o_p
 * (a part with lse_p = -inf counts for nothing; all -inf gives o = 0, lse = -inf).
 *   o_parts [parts, rows, n_heads_q, head_dim] bf16; lse_parts [parts, rows, n_heads_q] fp32
 *   o [rows, n_heads_q, head_dim] bf16; lse [rows, n_heads_q] fp32 or NULL
 */
qsa_status qsa_merge_attn_states(const qsa_config *cfg, const qsa_bf16 *o_parts, const float *lse_parts,
                                 int32_t parts, int64_t rows, qsa_bf16 *o, float *lse, void *stream);

/*
 * Sparse GQA attention, decode, with library-held scratch instead of a caller
 * workspace.  Computes exactly what qsa_sparse_attn_decode computes, with the
 * same schedule, and takes the same arguments minus ws / ws_bytes.
 * The reading notes describe no counterpart of this call: it exists for
 * callers that cannot allocate device memory at decode time, e.g. a serving
 * loop whose pool has reserved all free device memory up front, or a plain C
 * host with no device allocator of its own to hand a workspace from.
 *
 * Scratch: a fixed array of QSA_STATIC_SCRATCH_BYTES in the library's device
 * image; every GPU that loads libqsa.so holds it until the process exits.  The
 * call allocates and frees nothing (no cudaMalloc / cudaFree, no allocating
 * library routine).  The first call on a device, with that device current,
 * looks up the array's device address once (cudaGetSymbolAddress); make that
 * first call before any stream capture.
 * Sharing: every call on a device uses the SAME array, so two calls whose
 * kernels overlap on the GPU (different streams without ordering between them,
 * or concurrent host threads) race and corrupt each other's results; order
 * them on one stream.  Nothing in the array has to start at zero: each call
 * writes every partial state before the merge reads it.
 * Limit: a call whose partial softmax states need more than
 * QSA_STATIC_SCRATCH_BYTES returns QSA_ERR_SCRATCH_LIMIT before launching
 * anything (use qsa_sparse_attn_decode with a workspace there).  With 148 SMs
 * the partial states take (batch + 148) x 24.7 KB below batch 296 and nothing
 * from there on, 10.9 MB at most, so no batch size reaches the limit on B200.
 */
#define QSA_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)
qsa_status qsa_sparse_attn_decode_static_scratch(const qsa_config *cfg, const qsa_bf16 *q,
                                                 const qsa_bf16 *k_cache, const qsa_bf16 *v_cache,
                                                 const int32_t *cu_seqlens_k, int32_t batch,
                                                 int64_t total_k, const int32_t *sel, qsa_bf16 *o,
                                                 float *lse, void *stream);

/*
 * Decode with multi-token prediction.  The reading notes' decode measurement
 * ("结果 2") verifies next_n = 4 tokens per sequence per step (three MTP
 * prediction steps), and their section 5, step 5 says the MTP steps reuse the
 * QSA top-k indices.  Reading taken here: ONE selection per sequence serves its
 * next_n queries t = L - next_n .. L - 1 (L = cu_seqlens_k[s+1] - cu_seqlens_k[s],
 * the cache holding all next_n new tokens):
 *
 * qsa_index_select_mtp: the selection, from the indexer scores of the LAST query
 * (q_idx, w: [batch, n_heads_idx, idx_dim] / [batch, n_heads_idx], that query's).
 * Every query keeps its own trailing block (the budget sentence of section 6), so
 * the blocks floor((L - next_n) / r) .. floor((L - 1) / r) are all kept and the
 * other slots, at most k minus their number, go to the best blocks below the
 * first of them (ties to the lower index).  sel [batch, k] int32, ascending, -1
 * padded.  The scan and the exact rescoring are those of qsa_index_select's decode
 * rows.  1 <= next_n <= 4, k >= 2.  Workspace: qsa_workspace_size(cfg,
 * QSA_OP_INDEX_SELECT, batch, batch, max_len_k) bytes.
 *
 * qsa_sparse_attn_decode_mtp: the sparse attention of the next_n queries over the
 * shared selection, each cut to its own tokens j <= t (section 6).  One gathered
 * K/V tile serves every query of the sequence: the kernel puts the next_n x 24
 * (query, head) rows on the tensor cores' M side.
 *   q [batch, next_n, n_heads_q, head_dim] bf16; o the same shape;
 *   lse [batch, next_n, n_heads_q] fp32 or NULL; k_cache, v_cache packed as for
 *   qsa_sparse_attn_decode.
 * Workspace: qsa_workspace_size(cfg, QSA_OP_DECODE_MTP, batch, batch, 0) bytes
 * (partial softmax states when a sequence's tiles are split over several CTAs).
 */
qsa_status qsa_index_select_mtp(const qsa_config *cfg, const qsa_bf16 *q_idx, const float *w, const qsa_bf16 *kc,
                                int64_t kc_rows, const int32_t *cu_seqlens_k, const int32_t *cu_blocks,
                                int32_t batch, int32_t next_n, int64_t max_len_k, int32_t *sel, void *ws,
                                size_t ws_bytes, void *stream);
qsa_status qsa_sparse_attn_decode_mtp(const qsa_config *cfg, const qsa_bf16 *q, const qsa_bf16 *k_cache,
                                      const qsa_bf16 *v_cache, const int32_t *cu_seqlens_k, int32_t batch,
                                      int64_t total_k, int32_t next_n, const int32_t *sel, qsa_bf16 *o, float *lse,
                                      void *ws, size_t ws_bytes, void *stream);

/*
 * Dense causal GQA attention (the baseline the pages measure QSA against):
 * query t attends to every key j <= t of its sequence.  Same layouts as the
 * sparse prefill.  max_len_q and max_len_k are host bounds of L_q,s and L_k,s.
 * max_len_q == 1 (one query per sequence, decode) runs split-K flash decoding
 * over all blocks and needs qsa_workspace_size(cfg, QSA_OP_DENSE, batch,
 * total_q, max_len_k) bytes of workspace; otherwise no workspace (ws may be NULL).
 */
qsa_status qsa_dense_attn_prefill(const qsa_config *cfg, const qsa_bf16 *q, const qsa_bf16 *k,
                                  const qsa_bf16 *v, const int32_t *cu_seqlens_q,
                                  const int32_t *cu_seqlens_k, int32_t batch, int64_t total_q,
                                  int64_t total_k, int32_t max_len_q, int64_t max_len_k,
                                  qsa_bf16 *o, float *lse, void *ws, size_t ws_bytes, void *stream);

/* Workspace bytes an op needs (0 = none).  rows = query rows of the call,
 * max_len_k = longest key sequence.  Host only, no CUDA calls. */
size_t qsa_workspace_size(const qsa_config *cfg, int32_t op, int32_t batch, int64_t rows,
                          int64_t max_len_k);

/* Static string for a status code. */
const char *qsa_status_string(qsa_status status);

/* Synchronises `stream`, then copies the current device's sticky status word
 * into *status (QSA_OK if no kernel flagged an error); clear != 0 resets it. */
qsa_status qsa_get_device_status(void *stream, int32_t *status, int32_t clear);

/* ABI version (major * 100 + minor). */
int32_t qsa_version(void);

/* Fault injection for the failure-path tests.  Only a library built with
 * QSA_DEBUG_CHECKS (libqsa_debug.so: mbarrier waits limited to 20 ms) acts on
 * it; the release library returns QSA_ERR_UNSUPPORTED and changes nothing.
 *   site 0  no fault (the default)
 *   site 1  the decode scan's producer (qsa_index_select, decode rows) issues no
 *           copies for the second kc tile of each CTA, so the consumer's bounded
 *           wait runs out: the call's kernels return, the status word reads
 *           QSA_ERR_TIMEOUT and the next call without the fault runs normally.
 * Host only (one device-symbol copy); not thread-safe with calls in flight. */
qsa_status qsa_debug_inject(int32_t site);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H */
