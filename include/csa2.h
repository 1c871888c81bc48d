/*
 * csa2.h -- C ABI of the CSA2 step over an FP4 KV cache (B200, sm_100a).
 *
 * CSA2 ("Compressed Sparse Attention 2") as described for DeepSeek-V4.1-Flash:
 * every layer attends over 512 indices chosen by a lightweight indexer plus a
 * 128-token sliding window; layers run in one of three static modes (Full,
 * Reindex, Reuse) that share the main KV and the indexer keys across layers;
 * the main KV is stored as E2M1 codes with one E4M3 scale per 16 channels
 * (agentnet.co.il, "דיפסיק משיקה את V4.1-פלאש ...", sections "CSA2: דחיסה
 * לאורך ציר השכבות" and "קוונטיזציה ופריסה: FP4 ו-DRAM במקום SSD"; ai-wave.ru,
 * "DeepSeek V4.1-Flash: 1M контекст, FP4 KV-кэш ...", second to fourth
 * paragraphs).
 *
 * Conventions for every call
 * --------------------------
 * - All tensor arguments are DEVICE pointers owned by the caller; the library
 *   allocates no memory.  Scratch space comes from a caller workspace sized by
 *   csa2_workspace_bytes(), except in csa2_indexer_score_topk_noalloc, whose
 *   scratch is one static device array of CSA2_NOALLOC_SCRATCH_BYTES that the
 *   library holds on every GPU that loads it.
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *   default stream) and performs no host synchronisation and no allocation;
 *   csa2_check_device_error() is the only call that synchronises.  The calls
 *   that take their scratch from a caller workspace, and those that need no
 *   scratch, can be captured in a CUDA graph.
 * - bf16 tensors are passed as uint16_t bit patterns.
 * - Return value: CSA2_OK or a csa2_status error.  Argument, shape, alignment,
 *   workspace and mode-order errors are detected on the host before anything is
 *   launched (nothing is enqueued then).  Out-of-range page ids, positions or
 *   sequence ids found by a kernel are not faults: the kernel skips that row,
 *   ORs a CSA2_DEVERR_* bit into cache->error_word, and the host sees it through
 *   csa2_check_device_error().
 *
 * Cache layout in HBM (all pools indexed by the same page id)
 * ----------------------------------------------------------
 * - kv_pool:       page p holds 64 token rows of 288 B at p*18432 + slot*288.
 *                  Row = 256 B of E2M1 codes (channel 2j in the low nibble of
 *                  byte j, channel 2j+1 in the high nibble) followed by 32 E4M3
 *                  scale bytes (scale g covers channels 16g..16g+15).
 * - idxk_pool:     page p holds 64 indexer keys.  CSA2_IDXK_BF16: bf16
 *                  [64][64], 8192 B/page.  CSA2_IDXK_FP8: E4M3 codes
 *                  [64][64] (byte d = dimension d) followed by the 64 fp32
 *                  scales, 4352 B/page; key = scale x code.
 * - blockkey_pool: page p holds the 8 block keys of its 8-token blocks,
 *                  bf16 [8][64], 1024 B/page.
 * - page_table[b*max_pages + i] = page id of tokens 64i..64i+63 of sequence b.
 * Positions are entry positions (after 2:1 compression, for ratio-2 caches).
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* csa2_stream_t; /* == cudaStream_t */

/* ---- constants of the method ---- */
#define CSA2_LATENT_DIM 512       /* channels of the shared K = V latent            */
#define CSA2_SCALE_GROUP 16       /* channels per E4M3 scale                        */
#define CSA2_ROW_BYTES 288        /* 256 code bytes + 32 scale bytes per token      */
#define CSA2_PAGE_TOKENS 64
#define CSA2_IDX_HEADS 4          /* indexer query heads                            */
#define CSA2_IDX_DIM 64           /* indexer head dim == shared indexer key dim     */
#define CSA2_BLOCK_TOKENS 8       /* tokens per indexer block                       */
#define CSA2_POOL_BLOCKS 2048     /* blocks in the hierarchical candidate pool      */
#define CSA2_TOP_K 512            /* indices selected per query                     */
#define CSA2_WINDOW 128           /* sliding-window length                          */
#define CSA2_REPLAY 128           /* tokens recomputed by bounded replay            */
#define CSA2_HIER_FLAT 0          /* indexer: every visible entry is a candidate    */
#define CSA2_HIER_MEAN 1          /* pool of 2,048 blocks by mean-pooled block keys  */
#define CSA2_HIER_MAX 2           /* pool by the largest token score of each block   */
#define CSA2_IDXK_BF16 0          /* indexer keys stored as bf16, 128 B per token   */
#define CSA2_IDXK_FP8 1           /* 64 E4M3 codes + one fp32 scale, 68 B per token */

typedef enum {
  CSA2_OK = 0,
  CSA2_ERR_INVALID_ARG = 1,   /* NULL pointer, bad enum, negative count       */
  CSA2_ERR_SHAPE = 2,         /* unsupported size (heads, compress, ...)      */
  CSA2_ERR_ALIGNMENT = 3,     /* pointer not 16-byte aligned where required   */
  CSA2_ERR_MODE_STATE = 4,    /* layer modes called out of order              */
  CSA2_ERR_WORKSPACE = 5,     /* workspace missing or too small               */
  CSA2_ERR_CUDA = 6,          /* a CUDA launch or runtime call failed         */
  CSA2_ERR_DEVICE_BOUNDS = 7  /* a kernel found an out-of-range id (see bits) */
} csa2_status;

typedef enum { CSA2_FULL = 0, CSA2_REINDEX = 1, CSA2_REUSE = 2 } csa2_mode;

typedef enum {
  CSA2_OP_INDEXER = 1,
  CSA2_OP_ATTENTION = 2,
  CSA2_OP_SHARD_INDEXER = 3,    /* csa2_shard_indexer_candidates: nq, max_visible         */
  CSA2_OP_SHARD_MERGE = 4,      /* csa2_shard_merge_topk: nq, heads = nshard,
                                   max_visible = candidates per shard                     */
  CSA2_OP_SHARD_ATTENTION = 5   /* csa2_sparse_attn_shard: nq, heads                      */
} csa2_op;

/* bits OR-ed into *error_word by kernels */
#define CSA2_DEVERR_PAGE 1u  /* page id outside [0, n_pages) or page slot >= max_pages */
#define CSA2_DEVERR_POS 2u   /* position/index outside the sequence's visible length   */
#define CSA2_DEVERR_SEQ 4u   /* sequence id outside [0, batch)                         */
#define CSA2_DEVERR_TIMEOUT 8u  /* a bounded wait for tensor-core completion ran out    */

/* Paged cache; every pointer is device memory owned by the caller. */
typedef struct {
  void* kv_pool;              /* n_pages * 18432 B, 16-B aligned               */
  void* idxk_pool;            /* n_pages * 8192 B (bf16 keys) or * 4352 B (FP8
                                 keys), 16-B aligned                           */
  void* blockkey_pool;        /* n_pages * 1024 B, 16-B aligned                */
  int64_t n_pages;            /* 1 .. 2^25 (attention names rows by 31 bits)   */
  const int32_t* page_table;  /* int32 [batch][max_pages]                      */
  int32_t max_pages;
  int32_t batch;              /* 1 .. 2^23                                     */
  const int32_t* seq_lens;    /* int32 [batch]: entries present per sequence   */
  uint32_t* error_word;       /* one uint32, zeroed by the caller              */
  uint64_t cache_id;          /* caller-chosen identity used by mode checks    */
  void* swa_rows;             /* optional separate sliding-window store, NULL:
                                 none (the window is read from kv_pool); else
                                 [batch][128][288 B] FP4 rows, 16-B aligned,
                                 position p of sequence b in slot p % 128      */
  int32_t idxk_format;        /* CSA2_IDXK_BF16 (0) or CSA2_IDXK_FP8           */
} csa2_cache;

/* Index sets produced by the indexer and consumed by attention.  Device
 * buffers are caller-owned; the tags are host-side state kept by the library
 * to enforce the Full -> Reindex -> Reuse order. */
typedef struct {
  int32_t* idx;          /* int32 [rows][512]: positions, ascending, -1 padded      */
  int32_t* pool_blocks;  /* int32 [rows][2048]: candidate blocks, ascending, -1 pad */
  int32_t rows;          /* capacity in queries                                     */
  int32_t layer;         /* layer whose indexer call last wrote idx (-1: none)      */
  int32_t mode;          /* CSA2_FULL or CSA2_REINDEX: mode of that call            */
  int32_t pool_layer;    /* layer whose hierarchical Full call wrote pool_blocks    */
  uint64_t cache_id;     /* cache the sets were computed on                         */
  int32_t nq;            /* queries written by the last indexer call                */
  int32_t* attn_rows;    /* optional int32 [rows][CSA2_ATTN_ROWS_INTS] (NULL: none):
                            attended rows resolved by the last Full / Reindex
                            attention call, reused by Reuse calls                   */
  int32_t rows_layer;    /* layer of the attention call that wrote attn_rows (-1)   */
  int32_t rows_split;    /* row ranges per query of that call                       */
  int32_t rows_nq;       /* queries of that call                                    */
} csa2_indexset;

/* int32 per query of an index set's attention row cache: 640 physical row ids
 * (page * 64 + slot, in the order attention visits them) and 8 range counts. */
#define CSA2_ATTN_ROWS_INTS 648

/* Reset an index set's tags (no device work). */
void csa2_indexset_init(csa2_indexset* set, int32_t* idx, int32_t* pool_blocks, int32_t rows);

/* Attach (or, with NULL, detach) a caller-owned device buffer of
 * rows * CSA2_ATTN_ROWS_INTS int32 (4-B aligned) in which attention keeps the
 * physical rows it resolved.  A Full or Reindex csa2_sparse_attn call writes
 * them; a following Reuse call on the same set with the same queries (nq,
 * q_seq, q_visible) and the cache unchanged reads them instead of resolving
 * the selected positions and the window through the page table again.  Any
 * indexer call on the set discards them.  This is a schedule of the same
 * computation (the attended positions of a Reuse layer are those of the
 * latest Full / Reindex layer: agentnet.co.il, "CSA2: דחיסה לאורך ציר
 * השכבות"); it changes no result. */
void csa2_indexset_attach_rows(csa2_indexset* set, int32_t* attn_rows);

/*
 * csa2_kv_quant_append -- write new entries into the FP4 cache.
 *
 * Defines the main-KV codec (agentnet.co.il, section "קוונטיזציה ופריסה: FP4
 * ו-DRAM במקום SSD": E2M1 with one E4M3 scale per 16 channels, no global
 * scale) and the encoder's compression ratio 2 (same page, section "CSA2:
 * דחיסה לאורך ציר השכבות").  Entry i is built from input rows
 * [compress*i, compress*i + compress) of kv (bf16 [compress*n][512]) and idxk
 * (bf16 [compress*n][64]); with compress == 2 the pair is averaged in fp32.
 * Per group of 16 channels: scale = E4M3 nearest to amax/6 (ties to even,
 * saturating at 448); code = sign | E2M1 nearest to |x|/scale (ties to even,
 * saturating at 6); a zero scale stores code 0.  The entry is written at
 * position entry_pos[i] of sequence entry_seq[i] (both int32 [n]); the
 * indexer key is stored as bf16 (the fp32 pair mean rounded to nearest even
 * at ratio 2).  With CSA2_IDXK_FP8 that bf16 key k is stored quantised:
 * scale s = fl32(max_d |k_d| / 448), code_d = E4M3 nearest to fl32(k_d / s)
 * (ties to even, saturating at 448, sign kept), s == 0 stores zero codes; its
 * dequantised value is fl32(s x code).  The block key of every touched
 * 8-token block is recomputed as bf16(fp32 mean of the block's present
 * (dequantised) keys, ascending order).  seq_lens must already count the new entries (entry_pos[i] <
 * seq_lens[seq]).  kv and idxk must be 16-B aligned.  With a sliding-window
 * store (cache->swa_rows), entries among their sequence's last 128 positions
 * are also written to their slot there.
 */
int csa2_kv_quant_append(const csa2_cache* cache, const uint16_t* kv, const uint16_t* idxk,
                         const int32_t* entry_seq, const int32_t* entry_pos, int32_t n,
                         int32_t compress, csa2_stream_t stream);

/*
 * csa2_indexer_score_topk -- Full or Reindex indexer step.
 *
 * Defines the CSA2 indexer (agentnet.co.il, section "CSA2: דחיסה לאורך ציר
 * השכבות": Full selects 512 fresh indices; Reindex ranks the last Full
 * layer's indexer K with its own indexer Q; the decoder's hierarchical
 * indexer builds a pool of up to 2,048 blocks x 8 = 16,384 positions).
 * Query r (0 <= r < nq) has indexer query idx_q[r] (bf16 [4][64]), head
 * weights head_w[r] (float [4], or head_w == NULL for all ones), sequence
 * q_seq[r] and visible length q_visible[r] (or seq_lens[q_seq[r]] if
 * q_visible == NULL); max_visible >= every visible length (host-known bound
 * that sizes the grid and the workspace); nq <= 65535.
 * score(q, k) = sum_h w_h * max(0, q_h . k) in fp32; an FP8 key scores
 * s x score(q, code values).  Block keys are bf16 in both formats.
 *  - CSA2_FULL, hierarchical == CSA2_HIER_MEAN (decoder): if ceil(v/8) >
 *    2048 the 2,048 best block keys form the pool, else every block does;
 *    writes set->pool_blocks[r] and the 512 best pool tokens to set->idx[r].
 *  - CSA2_FULL, hierarchical == CSA2_HIER_MAX: the block score is the
 *    largest score of the block's present tokens (the pages do not fix the
 *    block score; this reading reads every key and loses nothing: the pool's
 *    512 best tokens are the 512 best of [0, v), which is how they are
 *    computed).  Writes the pool and set->idx[r] like CSA2_HIER_MEAN.
 *  - CSA2_FULL, hierarchical == CSA2_HIER_FLAT (encoder): 512 best of
 *    positions [0, v); no pool.
 *  - CSA2_REINDEX: 512 best tokens of the pool written by the last
 *    hierarchical Full call on `set` (requires set->pool_layer < layer).
 * Ranking: score descending, then position ascending; output ascending, -1
 * padded.  Workspace: csa2_workspace_bytes(CSA2_OP_INDEXER, nq, 0,
 * max_visible, hierarchical).  Sets set->layer = layer, set->mode = mode.
 */
int csa2_indexer_score_topk(const csa2_cache* cache, const uint16_t* idx_q, const float* head_w,
                            const int32_t* q_seq, const int32_t* q_visible, int32_t nq,
                            int64_t max_visible, int32_t mode, int32_t hierarchical,
                            int32_t layer, csa2_indexset* set, void* workspace,
                            size_t workspace_bytes, csa2_stream_t stream);

/*
 * csa2_sparse_attn -- CSA2 attention of one layer.
 *
 * Attended set of query r: the positions in set->idx[r] joined with the
 * window [max(0, v-128), v), each position once (128-token sliding window:
 * ai-wave.ru, second paragraph; agentnet.co.il, section "ארכיטקטורה שחותכת
 * בחצי את הפריפיל").  K = V = the decoded FP4 rows (every E2M1 x E4M3
 * product is exact in f16 and bf16); s = sm_scale * q . k; p = softmax over
 * the set; out[r] = sum p k, rounded to bf16.  The products run on the tensor
 * cores in f16 with fp32 accumulation: q is scaled by a power of two per
 * query (per group of its heads when a small batch splits the heads over
 * several clusters) so that it is exact in f16 down to 2^-28 of the largest
 * element it is scaled with, and the weights p are rounded to f16.  q: bf16 [nq][heads][512]; out: bf16 [nq][heads][512]; heads in
 * {16, 32, 48, 64}; nq <= 65535.  Mode checks (host): CSA2_FULL / CSA2_REINDEX need
 * set->layer == layer and set->mode == mode (the set is this layer's own);
 * CSA2_REUSE needs set->layer < layer (the latest Full or Reindex set).  An
 * empty set gives a zero output.  Workspace: csa2_workspace_bytes(
 * CSA2_OP_ATTENTION, nq, heads, 0, 0) (0 when a query's rows are not split
 * across CTAs; workspace may then be NULL).  With a row cache attached
 * (csa2_indexset_attach_rows), Full / Reindex calls record the resolved rows
 * in it (host tags rows_*) and Reuse calls read them.
 */
int csa2_sparse_attn(const csa2_cache* cache, const uint16_t* q, int32_t heads, float sm_scale,
                     const int32_t* q_seq, const int32_t* q_visible, int32_t nq, int32_t mode,
                     int32_t layer, csa2_indexset* set, uint16_t* out, void* workspace,
                     size_t workspace_bytes, csa2_stream_t stream);

/*
 * csa2_swa_replay -- bounded replay of the sliding window.
 *
 * On a cache miss only the last 128 tokens are recomputed (ai-wave.ru, second
 * paragraph; news.hamidun.com, section "Три механизма экономии памяти";
 * agentnet.co.il, section "ארכיטקטורה שחותכת בחצי את הפריפיל"), in the decoder
 * and in the encoder (same agentnet.co.il section: 128 tokens instead of
 * layers x window).  For every sequence b with L = seq_lens[b] entries: if
 * miss[b] != 0, entries [L - min(128, L), L) are re-encoded from the last
 * min(128, L) entries' raw rows of kv_last[b] (bf16 [batch][128 compress][512],
 * entry r of the block made of raw rows [compress r, compress r + compress),
 * averaged in fp32 when compress == 2) and idxk_last[b] (bf16
 * [batch][128 compress][64]); otherwise only entry L-1 is written, from the
 * block's last entry.  Same codec as csa2_kv_quant_append.  Without a
 * sliding-window store the rows, indexer keys and block keys of kv_pool are
 * rewritten; with one (cache->swa_rows) only its slots are rewritten -- the
 * window lives apart from the global cache (ai-wave.ru, fourth paragraph;
 * agentnet.co.il, section "קוונטיזציה ופריסה: FP4 ו-DRAM במקום SSD") -- and
 * idxk_last may be NULL.
 */
int csa2_swa_replay(const csa2_cache* cache, const uint16_t* kv_last, const uint16_t* idxk_last,
                    const uint8_t* miss, int32_t compress, csa2_stream_t stream);

/*
 * csa2_indexer_score_topk_noalloc -- csa2_indexer_score_topk without a
 * caller workspace, for callers that cannot allocate device memory (a host
 * framework that owns all device memory and gives plugins no allocator, a
 * serving loop that must never reach cudaMalloc, a fixed memory budget).
 *
 * The pages describe no such interface; it has no counterpart in the method.
 * Same arguments and results as csa2_indexer_score_topk minus the workspace:
 * the score buffer is a library-owned static device array of
 * CSA2_NOALLOC_SCRATCH_BYTES, present on every GPU that loads the library
 * until the process exits.  Argument and mode-order errors are reported as by
 * csa2_indexer_score_topk; a valid request whose workspace
 * (csa2_workspace_bytes) exceeds that size returns CSA2_ERR_WORKSPACE without
 * launching anything.
 * All calls share the one array: calls that overlap on the GPU race, so keep
 * them on one stream.  The array keeps the last call's contents; nothing in
 * it needs to start at zero.  The first call on a device looks up the
 * array's device address (a one-time set-up); make it before any stream
 * capture.  The address is kept for the life of the process, so the call is
 * not supported after cudaDeviceReset() on that device.  Allocates nothing.
 */
#define CSA2_NOALLOC_SCRATCH_BYTES (16u << 20)   /* 16 MiB */
int csa2_indexer_score_topk_noalloc(const csa2_cache* cache, const uint16_t* idx_q,
                                    const float* head_w, const int32_t* q_seq,
                                    const int32_t* q_visible, int32_t nq, int64_t max_visible,
                                    int32_t mode, int32_t hierarchical, int32_t layer,
                                    csa2_indexset* set, csa2_stream_t stream);

/* ------------------------------------------------------------------------
 * Position-sharded decode of long sequences (multi-GPU).
 *
 * A sequence is split into contiguous position ranges (shards), one per GPU;
 * a shard's cache holds its positions as entries 0 .. n-1 of its own
 * sequence, and shard_offset[r] (a multiple of 8) is the global position of
 * entry 0 for query r.  Per layer every GPU calls, with the same queries:
 *   1. csa2_shard_indexer_candidates(stage CSA2_SHARD_BLOCKS): its 2,048 best
 *      blocks (score, global block id); all-gather; csa2_shard_merge_topk
 *      (k = 2048) -> the global pool, identical on every GPU;
 *   2. csa2_shard_indexer_candidates(stage CSA2_SHARD_TOKENS, the pool): its
 *      512 best pool positions (score, global position); all-gather;
 *      csa2_shard_merge_topk (k = 512) -> the global index set;
 *   3. csa2_sparse_attn_shard: attention over the set's positions and the
 *      window's positions that it holds -> normalised output + base-2
 *      log-sum-exp; all-gather; csa2_shard_combine -> the layer's output.
 * Each merge is exact: an element of a global top-k is in its own shard's
 * top-k; candidate lists concatenated in shard order are in ascending global
 * order, so ties go to the lowest position as in the unsharded call.  The
 * result equals the unsharded hierarchical (mean-pooled) Full step up to the
 * rounding of the partial outputs (the pool, the 2,048-block rule and the
 * window are those of csa2_indexer_score_topk / csa2_sparse_attn; agentnet.co.il,
 * section "CSA2: דחיסה לאורך ציר השכבות").  The exchanges are the caller's
 * collectives (e.g. an NCCL all-gather); the merge and combine calls read the
 * gathered rows through (query_stride, shard_stride) in rows: shard s of
 * query q is row q * query_stride + s * shard_stride.
 * ------------------------------------------------------------------------ */
#define CSA2_SHARD_BLOCKS 0
#define CSA2_SHARD_TOKENS 1

/* Candidates of one shard for queries r < nq (sequence q_seq[r] of `cache`,
 * all its entries visible, idx_q / head_w as in csa2_indexer_score_topk).
 * stage CSA2_SHARD_BLOCKS: cand_score / cand_id [nq][2048] = the shard's
 * 2,048 best block keys, ids = global block ids (shard_offset / 8 + local),
 * ascending, (-inf, -1) padded.  stage CSA2_SHARD_TOKENS: global_pool
 * [nq][2048] (global block ids, -1 padded) -> cand_score / cand_id
 * [nq][512] = the 512 best positions of the pool blocks this shard holds,
 * global positions, ascending, (-inf, -1) padded.  Workspace:
 * csa2_workspace_bytes(CSA2_OP_SHARD_INDEXER, nq, 0, max_visible, 0).
 * A non-empty shard whose shard_offset is negative or not a multiple of 8
 * raises CSA2_DEVERR_POS. */
int csa2_shard_indexer_candidates(const csa2_cache* cache, const uint16_t* idx_q, const float* head_w,
                                  const int32_t* q_seq, const int32_t* shard_offset, int32_t nq,
                                  int64_t max_visible, int32_t stage, const int32_t* global_pool,
                                  float* cand_score, int32_t* cand_id, void* workspace,
                                  size_t workspace_bytes, csa2_stream_t stream);

/* Exact top-k of gathered candidate lists: for query q, the nshard rows of n
 * candidates (score, id) at rows q * query_stride + s * shard_stride (n a
 * multiple of 8; rows in shard order hold ascending ids, -1 entries with
 * -inf scores are no candidates).  Writes out_id [nq][k] (ascending, -1
 * padded) and, if out_score != NULL, their scores.  Workspace:
 * csa2_workspace_bytes(CSA2_OP_SHARD_MERGE, nq, nshard, n, 0). */
int csa2_shard_merge_topk(const float* cand_score, const int32_t* cand_id, int32_t nshard, int32_t nq,
                          int32_t n, int64_t query_stride, int64_t shard_stride, int32_t k,
                          int32_t* out_id, float* out_score, void* workspace, size_t workspace_bytes,
                          csa2_stream_t stream);

/* Attention of one shard: query r attends over the positions of global_idx[r]
 * (global positions, [nq][512], -1 padded) that this shard holds, joined with
 * the window positions [window_start[r], end) that it holds (window_start =
 * the global window's first position, max(0, L - 128)).  out (bf16
 * [nq][heads][512]) is normalised over that set; lse2 (float [nq][heads]) is
 * its base-2 log-sum-exp of sm_scale q . k (-inf, with a zero output, when
 * the shard holds none of the set).  Same numerics as csa2_sparse_attn.
 * Workspace: csa2_workspace_bytes(CSA2_OP_SHARD_ATTENTION, nq, heads, 0, 0). */
int csa2_sparse_attn_shard(const csa2_cache* cache, const uint16_t* q, int32_t heads, float sm_scale,
                           const int32_t* q_seq, const int32_t* shard_offset, const int32_t* global_idx,
                           const int32_t* window_start, int32_t nq, uint16_t* out, float* lse2,
                           void* workspace, size_t workspace_bytes, csa2_stream_t stream);

/* Merge of the shards' attention outputs: out[q] = sum_s w_s O_s / sum_s w_s,
 * w_s = 2^(lse2_s - max_s lse2_s), over the shards with lse2 > -inf (zero if
 * none), rounded to bf16.  part: bf16 rows of [heads][512] and lse2: rows of
 * [heads], shard s of query q at row q * query_stride + s * shard_stride. */
int csa2_shard_combine(const uint16_t* part, const float* lse2, int32_t nshard, int32_t nq, int32_t heads,
                       int64_t query_stride, int64_t shard_stride, uint16_t* out, csa2_stream_t stream);

/* Workspace bytes for an indexer call (op = CSA2_OP_INDEXER: nq, max_visible,
 * hierarchical), an attention call (op = CSA2_OP_ATTENTION: nq, heads) or a
 * sharded call (CSA2_OP_SHARD_*, arguments as listed with the ops).
 * Returns 0 for an invalid request or when none is needed. */
size_t csa2_workspace_bytes(int32_t op, int32_t nq, int32_t heads, int64_t max_visible,
                            int32_t hierarchical);

/* Synchronise `stream`, read and clear cache->error_word; *bits (may be NULL)
 * receives the CSA2_DEVERR_* bits.  Returns CSA2_ERR_DEVICE_BOUNDS if any bit
 * was set, CSA2_ERR_CUDA if the stream reported an error, else CSA2_OK. */
int csa2_check_device_error(const csa2_cache* cache, csa2_stream_t stream, uint32_t* bits);

/* Static description of a status code. */
const char* csa2_status_string(int status);

/* Library version (major*10000 + minor*100 + patch). */
int csa2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CSA2_H */
