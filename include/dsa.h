/*
 * dsa.h - C ABI of the B200 (sm_100a) DSA layer-group library (libdsa_b200.so).
 *
 * The method (prose sources):
 *   - "GLM 5.2: How Four Co-Designed Mechanisms Beat Raw Scale", section "DeepSeek Sparse
 *     Attention": Stage 1, coarse scoring (an indexer scores every token of the context for
 *     the current query); Stage 2, fine selection (the top-2,048 tokens get full attention).
 *   - same page, section "IndexShare: Amortizing the Indexer": the indexer runs once per
 *     block of 4 layers and the block shares its selection.
 *   - twiscan.com post on GLM-5.2 (IndexShare): the indexer runs in FP8; one indexer is
 *     shared by a group of 4 layers and the other 3 reuse its selection.
 *   - "GLM-5.3-Flash hybrid sparse-linear attention with IndexPool", section "What
 *     changed": IndexPool pools four indexer keys into one (factors 2 and 8 take the same
 *     mean over 2 or 8 keys).
 *
 * Conventions shared by every entry point
 *   Positions   Sequence b holds ctx_len[b] keys (rows 0..ctx_len[b]-1 of its caches) and T
 *               new queries at its end: query t sits at position pos(b,t) = ctx_len[b]-T+t.
 *               A key row s (or pooled block s when pool > 1) is visible to the query iff
 *               pool*s <= pos(b,t).  ctx_len is a DEVICE array of B int32, normally
 *               T <= ctx_len[b] <= S_max * pool; the scoring and selection kernels also
 *               accept values outside that range (a query at pos < 0 sees no key, and only
 *               the S_max rows present are ever visible), which the key-sharded form below
 *               relies on.
 *   Types       e4m3 = OCP FP8 E4M3 ("e4m3fn") codes stored as uint8, unit scale.
 *               bf16 = bfloat16 stored as uint16.  Scores and weights are IEEE fp32.
 *   Layouts     Row-major, innermost dimension last, as written in each comment.
 *   Memory      Every pointer is a device pointer (unless stated) owned by the caller.  The
 *               library allocates no memory; calls that need scratch take a caller
 *               workspace and say how large it must be.  Pointers must be 16-byte aligned
 *               and row strides multiples of 16 bytes.
 *   Streams     `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *               Every call only enqueues work on that stream; none synchronises the host.
 *   Errors      Every call returns a dsa_status.  On any non-zero status nothing was
 *               enqueued (argument checks happen before the first launch), except
 *               DSA_ERR_CUDA from a failed launch, after which dsa_last_cuda_error() gives
 *               the cudaError_t.  Unsupported shapes are rejected, never emulated.
 *   Threads     Calls are reentrant; concurrent calls must not share output or workspace
 *               buffers.
 */
#ifndef DSA_B200_H
#define DSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,         /* null pointer, negative or inconsistent size */
  DSA_ERR_UNSUPPORTED_SHAPE = 2,   /* a head count / dim / k outside the supported set */
  DSA_ERR_MISALIGNED = 3,          /* pointer or stride not 16-byte aligned */
  DSA_ERR_WORKSPACE_TOO_SMALL = 4, /* ws_bytes below the size the *_workspace_size call gives */
  DSA_ERR_CUDA = 5,                /* a CUDA launch failed; see dsa_last_cuda_error() */
  DSA_ERR_TIMEOUT = 6,             /* a bounded device-side wait gave up (kernel exited early) */
  DSA_ERR_INDEX_RANGE = 7          /* an attention call met a selected id >= its S_kv (skipped) */
} dsa_status;

/* Static, NUL-terminated description of a status code (thread-safe). */
const char* dsa_status_string(int status);

/* cudaError_t of the last failed launch on the calling thread (0 if none). */
int dsa_last_cuda_error(void);

/* Number of the library's kernel launches enqueued by the calling thread so far
 * (a running counter, for accounting in benchmarks). */
uint64_t dsa_launch_count(void);

/* Synchronises `stream`, then reads and clears the device status words of the library's
 * kernels on the current device.  Returns DSA_OK; DSA_ERR_TIMEOUT when a kernel gave up one
 * of its bounded waits since the last call (that launch exited early and its outputs are
 * incomplete); else DSA_ERR_INDEX_RANGE when an attention launch met a selected id at or
 * beyond its S_kv (that id was skipped like a -1, and nothing outside the cache was read);
 * or DSA_ERR_CUDA if the synchronisation failed.  Every wait inside the tensor-core kernels
 * has a time limit, so no launch can hang. */
int dsa_device_status(void* stream);

/* Test hook for the failure path: enqueues one thread that waits, through the kernels' own
 * bounded wait, on a barrier that nothing ever completes, so the wait gives up after
 * limit_ns (1 ns .. 1 s) and sets the device status word; the next dsa_device_status() then
 * returns DSA_ERR_TIMEOUT.  Faults nothing; the CUDA context stays usable. */
int dsa_debug_wait_timeout(uint64_t limit_ns, void* stream);

/* Test hook for the real kernels' failure paths: sets the time limit of every bounded wait in
 * the tensor-core indexer and attention kernels on the current device (1 ns .. 2 s; 0 restores
 * the default of 2 s; below 1 us, every wait that is not ready at its first non-blocking check
 * gives up at once).  Synchronous (a copy to device memory); calls whose kernels are in flight
 * keep the limit they read.  With a limit shorter than a normal wait, a launch gives up early,
 * drains its copies and MMAs, frees TMEM and returns: dsa_device_status() then returns
 * DSA_ERR_TIMEOUT and that launch's outputs are incomplete; the context stays usable. */
int dsa_debug_set_wait_limit(uint64_t limit_ns);

/* ------------------------------------------------------------------------------------
 * Paged caches (optional on every call that reads a cache; NULL = contiguous per sequence).
 * The serving form of decode and chunked prefill: every cache the call reads (indexer keys
 * k_idx, latent/K rows kv, separate V rows v) is a pool of num_pages pages of page_size rows
 * shared by all sequences, and logical row s of sequence b is physical row
 *     block_table[b * pages_per_seq + s / page_size] * page_size + s % page_size
 * of each pool (k_idx: rows of d_I bytes; kv and v: rows at the call's row strides; their
 * batch strides are unused).  A sequence holds up to pages_per_seq * page_size logical rows,
 * which bounds S_max and S_kv.  page_size is a power of two >= 128, so a key tile of the
 * indexer never straddles a page.  block_table is a DEVICE array [B, pages_per_seq] of int32
 * page ids in [0, num_pages); an id outside that range is never followed (the indexer reads
 * zeros in its place, the attention skips the row) and dsa_device_status() then returns
 * DSA_ERR_INDEX_RANGE.
 * ------------------------------------------------------------------------------------ */
typedef struct dsa_paging {
  const int32_t* block_table;   /* device [B, pages_per_seq] int32 page ids */
  int32_t page_size;            /* rows per page: a power of two >= 128 */
  int32_t pages_per_seq;        /* columns of block_table */
  int32_t num_pages;            /* pages in each pool */
} dsa_paging;

/* ------------------------------------------------------------------------------------
 * dsa_index_scores - the lightning indexer (Stage 1, coarse scoring; FP8 per the
 * IndexShare post).  For every query t in [t_begin, t_begin + t_count) of every sequence:
 *
 *     I[t,s] = sum_{j<H_I} w[t,j] * max(0, sum_{d<d_I} q_idx[t,j,d] * k_idx[s,d])
 *
 * over the visible key rows s (pool*s <= pos(b,t)).  FP8 products are exact in fp32;
 * accumulation is fp32 on the tensor cores; the weighted ReLU reduction runs in fp32 in
 * the epilogue, so the per-head logits never reach memory.
 *
 *   q_idx  [B, T, H_I, d_I] e4m3      w [B, T, H_I] fp32      k_idx [B, S_max, d_I] e4m3
 *   scores [B, t_count, ld] fp32 out:  row (b, t - t_begin); entries s < n_valid hold I;
 *          entries from n_valid up to the end of the 128-key tile that holds the last
 *          visible key are -inf; entries beyond are not written.
 *   pool   1, or 2, 4 or 8 when k_idx holds IndexPool blocks (validity pool*s <= pos).
 *   paging NULL, or the page pool k_idx is (pool == 1 only; see dsa_paging).
 * Supported: (H_I, d_I) in {(4, 64), (64, 128)}; ld >= S_max, ld % 4 == 0.
 * ------------------------------------------------------------------------------------ */
int dsa_index_scores(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                     const int32_t* ctx_len, int B, int T, int S_max, int H_I, int d_I,
                     int pool, int t_begin, int t_count, float* scores, int64_t ld,
                     const dsa_paging* paging, void* stream);

/* ------------------------------------------------------------------------------------
 * dsa_topk - Stage 2, fine selection: per query row, the k_eff = min(k, n_valid) keys with
 * the largest scores, n_valid = min(S_max, pos/pool + 1).  Ties at the k-th score are
 * broken toward lower key index.  The selected keys are written in ascending key order,
 * followed by -1 padding.  With pool > 1 (IndexPool) the k selected blocks expand to
 * pool*k token ids pool*blk .. pool*blk+pool-1 (ascending); tokens beyond pos become -1.
 *
 *   scores  [B, t_count, ld] fp32 (as written by dsa_index_scores for the same t_begin)
 *   idx     [B, T, k*pool] int32 out; rows t_begin .. t_begin+t_count-1 are written.
 * Supported: 1 <= k <= 2048, pool in {1, 2, 4, 8}, ld % 4 == 0.
 * ------------------------------------------------------------------------------------ */
int dsa_topk(const float* scores, int64_t ld, const int32_t* ctx_len, int B, int T, int S_max,
             int pool, int t_begin, int t_count, int k, int32_t* idx, void* stream);

/* ------------------------------------------------------------------------------------
 * dsa_index_select - Stage 1 and Stage 2 together: the selection dsa_index_scores followed by
 * dsa_topk would give for rows t_begin .. t_begin+t_count-1 (same arguments, same ids bit for
 * bit), without writing the full score rows when the keys allow it ("fused": contiguous keys,
 * S_max a multiple of 16):
 *   1. the indexer scores every 16th key row; per query row the r-th largest of those samples
 *      (r = k/8 clamped to [32, 512]) becomes the row's threshold tau;
 *   2. the indexer scores every visible key and appends only the keys scoring >= tau, as
 *      (score, key id), to a candidate row of up to 8192 entries;
 *   3. the exact top-k (ties toward lower key index, ids ascending) runs on the candidates:
 *      with at least k candidates, every key that the full row's top-k keeps is among them.
 *   Rows left with fewer than k candidates, or more than 8192, are redone from full score rows
 *   by a repair pass that runs only their work items.
 * Otherwise (paged keys, or S_max not a multiple of 16) the full score rows go through the
 * workspace.  k_idx: keys, or pooled blocks when pool > 1, as for dsa_index_scores.
 *   idx  [B, T, k*pool] int32 out (rows t_begin .. t_begin+t_count-1 written)
 *   ws   at least dsa_index_select_workspace_size(B, 1, S_max, pool) bytes; the call works in
 *        query chunks of the largest size that fits.
 * Supported: as dsa_index_scores, and 1 <= k <= 2048.
 * ------------------------------------------------------------------------------------ */
size_t dsa_index_select_workspace_size(int B, int t_chunk, int S_max, int pool);
int dsa_index_select(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                     const int32_t* ctx_len, int B, int T, int S_max, int H_I, int d_I, int pool,
                     int t_begin, int t_count, int k, int32_t* idx, void* ws, size_t ws_bytes,
                     const dsa_paging* paging, void* stream);

/* ------------------------------------------------------------------------------------
 * dsa_sparse_attn - attention of every query over its selected keys only (Stage 2; the
 * "China's First Frontier Model?" page, section "The Time has Come": attend only to the
 * indexer's candidates).  All Hq query heads share one KV head (MQA; MLA latent form when
 * V aliases the first d_v columns of the K row):
 *
 *     O[t,h,:] = sum_i p_i * V[idx[t,i], :],  p = softmax_i(sm_scale * q[t,h,:] . K[idx[t,i], :])
 *     lse[t,h] = log sum_i exp(sm_scale * q[t,h,:] . K[idx[t,i], :])
 *
 * bf16 inputs, fp32 online softmax and accumulation, bf16 output.  Entries idx < 0 are
 * skipped; a repeated index counts once per occurrence.  A row with no selected key gives
 * O = 0 and lse = -inf.
 *
 *   q    [B, T, Hq, d_qk] bf16 (contiguous)
 *   kv   K rows: element (b, s, c) at kv[b*kv_batch_stride + s*kv_row_stride + c], c < d_qk
 *   v    V rows, same form with v_* strides; NULL means V = the first d_v columns of kv
 *   S_kv rows per sequence in the K/V caches (>= 1).  The kernels check every selected id on
 *        the device: an id >= S_kv is skipped like a -1 (nothing outside the cache is read)
 *        and the next dsa_device_status() returns DSA_ERR_INDEX_RANGE.
 *   idx  [B, T, k] int32, entries in [0, S_kv) (normally [0, ctx_len[b])) or < 0
 *   out  [B, T, Hq, d_v] bf16          lse  [B, T, Hq] fp32 or NULL
 *   ws   scratch of at least dsa_sparse_attn_workspace_size(B, T, Hq, d_v, k) bytes
 *        (zero for long prefill; split-key partials for few-query batches such as decode)
 *   paging NULL, or the page pools kv (and v) are (see dsa_paging; S_kv <= its capacity)
 * Supported: (Hq, d_qk, d_v) in {(16, 128, 128), (128, 576, 512)}; 1 <= k <= 8192.
 * ------------------------------------------------------------------------------------ */
size_t dsa_sparse_attn_workspace_size(int B, int T, int Hq, int d_v, int k);
int dsa_sparse_attn(const uint16_t* q, const uint16_t* kv, const uint16_t* v,
                    int64_t kv_row_stride, int64_t kv_batch_stride, int64_t v_row_stride,
                    int64_t v_batch_stride, int S_kv, const int32_t* idx, int B, int T, int Hq, int d_qk,
                    int d_v, int k, float sm_scale, uint16_t* out, float* lse, void* ws,
                    size_t ws_bytes, const dsa_paging* paging, void* stream);

/* ------------------------------------------------------------------------------------
 * dsa_sparse_attn_noalloc - dsa_sparse_attn for callers that can neither allocate device
 * memory nor pass a workspace (for example an operator inside a runtime that owns all device
 * memory and offers its operators no scratch, or a serving loop that must not call cudaMalloc
 * once it runs).  The method described in the sources has no counterpart to this call: it is
 * a deployment variant.  Same arguments, layouts, checks and results as dsa_sparse_attn minus
 * `ws`; the split-key partials go to a fixed scratch array inside the library instead.
 *   - The scratch is dsa_noalloc_scratch_bytes() (16 MiB) per GPU that loads the library,
 *     held until the process exits.  When the default key split of a problem would need more
 *     partials than that (see dsa_sparse_attn_workspace_size), the call runs at the largest
 *     split count whose partials fit, down to one split, which needs no scratch: no problem
 *     is rejected for its size, larger ones only spread over fewer CTAs.
 *   - The first call on a device looks up the scratch's device address (with that device
 *     current) and caches it; make that first call before any stream capture.  A
 *     cudaDeviceReset() invalidates the cached address.
 *   - All calls on a device share the scratch: calls whose kernels may overlap on the GPU
 *     (other streams, other host threads) race on it and must be serialised by the caller.
 *     Nothing in the scratch needs to start at zero; a call ignores what the last one left.
 *   - Allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 * ------------------------------------------------------------------------------------ */
size_t dsa_noalloc_scratch_bytes(void);
int dsa_sparse_attn_noalloc(const uint16_t* q, const uint16_t* kv, const uint16_t* v,
                            int64_t kv_row_stride, int64_t kv_batch_stride, int64_t v_row_stride,
                            int64_t v_batch_stride, int S_kv, const int32_t* idx, int B, int T, int Hq,
                            int d_qk, int d_v, int k, float sm_scale, uint16_t* out, float* lse,
                            const dsa_paging* paging, void* stream);

/* ------------------------------------------------------------------------------------
 * dsa_index_pool - IndexPool ("What changed": four indexer keys pooled into one):
 *     k_pool[b, g, :] = e4m3(((k[4g] + k[4g+1]) + (k[4g+2] + k[4g+3])) * 0.25)
 * and for pool = 2 or 8 the same mean over 2 or 8 keys (a balanced pairwise sum times
 * 1/pool).  The sum runs in fp32 on the decoded keys and is exact there, so the requantisation
 * (round-to-nearest-even, saturating at +-448) is the only rounding.
 *   k_idx [B, S_max, d_I] e4m3 (or its page pool when paging != NULL)
 *   -> k_pool [B, S_max/pool, d_I] e4m3 (always contiguous).
 * Supported: pool in {2, 4, 8}, S_max % pool == 0, d_I % 16 == 0.
 * ------------------------------------------------------------------------------------ */
int dsa_index_pool(const uint8_t* k_idx, int B, int S_max, int d_I, int pool, uint8_t* k_pool,
                   const dsa_paging* paging, void* stream);

/* ------------------------------------------------------------------------------------
 * dsa_index_pool_tail - keeps a pooled key cache current as keys are appended (decode, chunked
 * prefill): for every sequence b it recomputes, exactly as dsa_index_pool does, the pooled
 * blocks that hold rows ctx_len[b]-T .. ctx_len[b]-1 (the keys this step appended; rows
 * outside [0, S_max) are ignored) and touches no other block.  So dsa_index_pool once, then
 * this call after every append, leaves k_pool equal to dsa_index_pool of the current cache at
 * the cost of the new rows alone.  A block the append leaves partly filled is pooled over the
 * rows the cache holds at that moment, as dsa_index_pool would pool it.  The method pools
 * blocks of consecutive keys and says nothing of how a serving system keeps them; this is the
 * plain incremental form of the same arithmetic.
 *   ctx_len device [B] int32 (after the append); T >= 1 rows appended per sequence.
 * Other arguments, layouts and support as for dsa_index_pool.
 * ------------------------------------------------------------------------------------ */
int dsa_index_pool_tail(const uint8_t* k_idx, const int32_t* ctx_len, int B, int T, int S_max, int d_I, int pool,
                        uint8_t* k_pool, const dsa_paging* paging, void* stream);

/* ------------------------------------------------------------------------------------
 * dsa_group_forward - one IndexShare group ("IndexShare: Amortizing the Indexer"): the
 * indexer and the top-k run ONCE, and each of the group_size attention layers reads the
 * same index buffer.  Equivalent to dsa_index_scores + dsa_topk over all queries (in query
 * chunks sized to the workspace; dsa_index_select instead when fused_select = 1), then
 * group_size x dsa_sparse_attn.
 * With pool > 1 the indexer runs on dsa_index_pool's blocks and `topk` counts blocks
 * (idx then holds pool*topk token ids per row).  The comparator without IndexShare is
 * group_size calls with group_size = 1 and per-layer indexer tensors.
 * ------------------------------------------------------------------------------------ */
typedef struct dsa_group_args {
  /* indexer, shared by the group */
  const uint8_t* q_idx;    /* [B, T, H_I, d_I] e4m3 */
  const float* w;          /* [B, T, H_I] fp32 */
  const uint8_t* k_idx;    /* [B, S_max, d_I] e4m3 */
  const int32_t* ctx_len;  /* device [B] */
  int32_t B, T, S_max, H_I, d_I;
  int32_t topk;            /* keys (pool 1) or blocks (pool > 1) selected per query */
  int32_t pool;            /* 1, or 2, 4 or 8 (IndexPool) */
  int32_t group_size;      /* attention layers sharing the selection, 1..16 */
  /* attention, one entry per layer: HOST arrays of group_size DEVICE pointers */
  const uint16_t* const* q;   /* [B, T, Hq, d_qk] bf16 */
  const uint16_t* const* kv;  /* K (latent) rows, strides below */
  const uint16_t* const* v;   /* NULL, or per-layer V (NULL entries alias kv) */
  uint16_t* const* out;       /* [B, T, Hq, d_v] bf16 */
  float* const* lse;          /* NULL, or per-layer [B, T, Hq] fp32 (NULL entries skip) */
  int64_t kv_row_stride, kv_batch_stride, v_row_stride, v_batch_stride;   /* elements; the same
                                                                             for every layer */
  int32_t Hq, d_qk, d_v;
  float sm_scale;
  int32_t* idx;            /* [B, T, topk*pool] int32 out: the shared selection */
  dsa_paging paging;       /* block_table NULL: contiguous caches; else k_idx and every
                              layer's kv (and v) are page pools sharing this table */
  int32_t fused_select;    /* 0 (default): full score rows + dsa_topk, the faster path on B200
                              (the indexer is tensor-bound, so its score rows cost little);
                              1: fused selection where the keys allow it (dsa_index_select) */
  const uint8_t* k_pooled; /* pool > 1 only.  NULL: the call pools k_idx into its workspace;
                              else the caller's pooled cache [B, S_max/pool, d_I] e4m3
                              (contiguous; dsa_index_pool, then dsa_index_pool_tail after each
                              append), which the indexer reads as is and no pooling runs */
} dsa_group_args;

/* Workspace for dsa_group_forward when the indexer is run over chunks of t_chunk queries
 * (t_chunk >= 1; larger chunks mean fewer launches).  dsa_group_forward uses the largest
 * chunk that fits in the ws_bytes it is given. */
size_t dsa_group_workspace_size(const dsa_group_args* args, int t_chunk);
int dsa_group_forward(const dsa_group_args* args, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * Context parallelism: the key caches sharded over ranks, rank r holding the contiguous key
 * rows [s0_r, s0_r + len_r) of every sequence.  The pages describe no multi-GPU form; this is
 * the exchange form of the same selection ("DeepSeek Sparse Attention", Stage 2: the top-k of
 * the whole row) and attention ("The Time has Come": attend only to the selected tokens).  Per
 * rank and query chunk:
 *   1. dsa_index_scores and dsa_topk over the rank's shard (S_max = len_r), with ctx_len - s0
 *      as the context lengths: positions and the causal rule then refer to the shard's own
 *      rows (a shard wholly after a query's position selects nothing for it, one wholly
 *      before it offers all its rows);
 *   2. dsa_gather_selected: the shard's selection as (score, global id) candidates;
 *   3. the caller all-gathers the candidates of every rank (e.g. NCCL all_gather);
 *   4. dsa_topk_merge: the exact top-k of the union, the ids dsa_topk would give over the
 *      whole row, identical on every rank;
 *   5. per layer: dsa_idx_localize, then dsa_sparse_attn over the rank's rows (want lse);
 *   6. the caller all-gathers every rank's (O, lse); dsa_attn_combine merges them.
 * A rank whose shard is empty (len_r = 0) calls nothing in steps 1, 2 and 5: it contributes
 * (-inf, -1) candidates and a part with O = 0, lse = -inf, which the merges ignore.
 * pool must be 1.  Errors and asynchrony as for the other calls.
 * ------------------------------------------------------------------------------------ */

/* Candidates of a shard's selection: for rows t_begin .. t_begin+t_count-1 of
 * idx [B, T, k] (ids local to the shard, from dsa_topk on scores [B, t_count, ld]),
 * cand_score/cand_id [B, t_count, k] = (scores[row][id], id + id_offset), or (-inf, -1) for a
 * -1 entry.  An id >= ld is skipped like a -1 (nothing past the score rows is read) and the
 * next dsa_device_status() returns DSA_ERR_INDEX_RANGE.  Supported: 1 <= k <= 2048. */
int dsa_gather_selected(const float* scores, int64_t ld, const int32_t* idx, int B, int T, int t_begin, int t_count,
                        int k, int32_t id_offset, float* cand_score, int32_t* cand_id, void* stream);

/* The exact top-k (ties toward lower key id, ids ascending, -1 padding) of the union of
 * n_parts shard selections: part p is cand_score/cand_id + p * part_stride, each
 * [B, t_count, kc] as dsa_gather_selected writes them (kc >= k).  The rows are those of
 * queries t_begin .. of a context of ctx_len[b] keys (S_total key rows per sequence); a row with
 * at most k visible keys selects them all.  idx [B, T, k] int32 out (rows t_begin.. written).
 * Candidate ids must be distinct within a row (disjoint shards).  An id >= the row's visible
 * key count is skipped, a row left with fewer than k candidates is written as all -1, and
 * either makes the next dsa_device_status() return DSA_ERR_INDEX_RANGE.
 * Supported: 1 <= k <= 2048, n_parts * kc <= 16384. */
int dsa_topk_merge(const float* cand_score, const int32_t* cand_id, int n_parts, int64_t part_stride, int kc,
                   const int32_t* ctx_len, int B, int T, int S_total, int t_begin, int t_count, int k, int32_t* idx,
                   void* stream);

/* out[i] = idx[i] - s0 when s0 <= idx[i] < s0 + s_len, else -1 (n entries): a selection of
 * global key ids as ids into the shard, for dsa_sparse_attn over the shard's rows. */
int dsa_idx_localize(const int32_t* idx, int64_t n, int32_t s0, int32_t s_len, int32_t* out, void* stream);

/* Merge of n_parts attention results over disjoint key sets: part_o [n_parts, rows, d_v] bf16
 * (each normalised over its keys, as dsa_sparse_attn writes it) and part_lse [n_parts, rows]
 * fp32 (-inf for a part with no keys) ->
 *     out[r] = sum_p exp(lse_p - lse) part_o[p][r],  lse[r] = log sum_p exp(lse_p)
 * as bf16 (lse may be NULL).  Supported: 1 <= n_parts <= 16, d_v even. */
int dsa_attn_combine(const uint16_t* part_o, const float* part_lse, int n_parts, int64_t rows, int d_v, uint16_t* out,
                     float* lse, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DSA_B200_H */
