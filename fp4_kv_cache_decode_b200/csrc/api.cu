// C ABI of the CSA2 library: host-side validation, mode-order checks and
// kernel launches.  No allocation, no host synchronisation (except in
// csa2_check_device_error); every launch goes to the caller's stream.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace csa2 {
cudaError_t launch_append(const CacheView&, const uint16_t*, const uint16_t*, const int32_t*,
                          const int32_t*, int, int, cudaStream_t);
cudaError_t launch_replay(const CacheView&, const uint16_t*, const uint16_t*, const uint8_t*,
                          int, cudaStream_t);
cudaError_t launch_score(int, const CacheView&, const uint16_t*, const float*, const int32_t*,
                         const int32_t*, const int32_t*, int, int64_t, int64_t, float*, float*, int64_t,
                         cudaStream_t);
cudaError_t launch_topk(int, const CacheView&, const float*, int64_t, const int32_t*, const int32_t*,
                        const int32_t*, int, int, int32_t*, int64_t, cudaStream_t, float* = nullptr,
                        const int32_t* = nullptr, int = 0, int = 1);
cudaError_t indexer_set_attributes();
cudaError_t launch_shard_localize(const CacheView&, const int32_t*, const int32_t*, const int32_t*, int, int,
                                  int32_t*, const int32_t*, int32_t*, int, cudaStream_t);
cudaError_t launch_shard_pack(const float*, const int32_t*, int, int, int64_t, int64_t, int, float*, int32_t*,
                              cudaStream_t);
cudaError_t launch_shard_combine(const uint16_t*, const float*, int, int, int, int64_t, int64_t, uint16_t*,
                                 cudaStream_t);
cudaError_t attention_set_attributes();
size_t attn_workspace_bytes(int nq, int H);
int attn_splits_for(int nq);
cudaError_t launch_attention(const CacheView&, const uint16_t*, int, float, const int32_t*,
                             const int32_t*, const int32_t*, int, uint16_t*, void*, int32_t*, int, int,
                             cudaStream_t, const int32_t* = nullptr, float* = nullptr);
}  // namespace csa2

using namespace csa2;

namespace {

constexpr int kSrcFlat = 0, kSrcBlockKeys = 1, kSrcPool = 2, kSrcCand = 3;
constexpr int32_t kMaxQueries = 65535;   // queries map to gridDim.y

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Kernel attributes (dynamic shared-memory opt-in) are per device: set once.
int ensure_device_setup() {
  static std::mutex mu;
  static bool done[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return CSA2_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    if (indexer_set_attributes() != cudaSuccess) return CSA2_ERR_CUDA;
    if (attention_set_attributes() != cudaSuccess) return CSA2_ERR_CUDA;
    done[dev] = true;
  }
  return CSA2_OK;
}

int make_view(const csa2_cache* c, CacheView* v) {
  if (c == nullptr) return CSA2_ERR_INVALID_ARG;
  if (!c->kv_pool || !c->idxk_pool || !c->blockkey_pool || !c->page_table || !c->seq_lens ||
      !c->error_word)
    return CSA2_ERR_INVALID_ARG;
  if (c->n_pages <= 0 || c->max_pages <= 0 || c->batch <= 0) return CSA2_ERR_SHAPE;
  if (c->idxk_format != CSA2_IDXK_BF16 && c->idxk_format != CSA2_IDXK_FP8) return CSA2_ERR_INVALID_ARG;
  // attention names a physical row by a 31-bit id (page x 64 + slot, or a
  // sliding-window slot batch x 128 + p % 128 under a flag bit)
  if (c->n_pages > ((int64_t)1 << 25) || c->batch > (1 << 23)) return CSA2_ERR_SHAPE;
  if (!aligned(c->kv_pool, 16) || !aligned(c->idxk_pool, 16) || !aligned(c->blockkey_pool, 16) ||
      !aligned(c->page_table, 4) || !aligned(c->seq_lens, 4) || !aligned(c->error_word, 4) ||
      !aligned(c->swa_rows, 16))
    return CSA2_ERR_ALIGNMENT;
  v->kv = static_cast<uint8_t*>(c->kv_pool);
  v->idxk = static_cast<uint8_t*>(c->idxk_pool);
  v->bk = static_cast<uint8_t*>(c->blockkey_pool);
  v->n_pages = c->n_pages;
  v->pt = c->page_table;
  v->max_pages = c->max_pages;
  v->batch = c->batch;
  v->seq_lens = c->seq_lens;
  v->err = c->error_word;
  v->swa = static_cast<uint8_t*>(c->swa_rows);
  v->idxk_fp8 = c->idxk_format == CSA2_IDXK_FP8 ? 1 : 0;
  return CSA2_OK;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Score-buffer stride (floats per query) of an indexer call.
// Long rows (more entries than one top-k CTA holds in registers) are selected
// in segments of kSegLen entries, one CTA each, whose nseg x k candidates
// (score, id) are merged by one more top-k -- exact, and ties still go to the
// lowest position since the segments' lists concatenate in ascending order.
// Used when the candidates fit one CTA and the rows alone would leave most SMs
// idle (fewer than kSegMaxRows queries: 4 x 1M decode rows go from 4 CTAs to 32);
// otherwise the streaming top-k runs (an 8,192-query prefill chunk already fills
// the GPU with one CTA per row, and segmenting it was measured slower).
constexpr int64_t kSegLen = 16384;
constexpr int kSegMaxRows = 256;

int seg_count(int64_t n_max, int k, int nq) {
  if (n_max <= kSegLen || nq >= kSegMaxRows) return 0;
  const int64_t nseg = (n_max + kSegLen - 1) / kSegLen;
  return nseg * k <= kSegLen ? (int)nseg : 0;
}

size_t seg_bytes(int nq, int64_t n_max, int k) {
  const int nseg = seg_count(n_max, k, nq);
  return nseg ? (size_t)nq * nseg * k * 8 : 0;
}

// Top-k of rows of up to n_max entries, segmented when seg_count() says so;
// cand: workspace for the segments' candidates (seg_bytes()).
cudaError_t select_topk(int src, const CacheView& v, const float* scores, int64_t stride, const int32_t* q_seq,
                        const int32_t* q_vis, const int32_t* pool, int nq, int k, int32_t* out,
                        int64_t out_stride, cudaStream_t s, int64_t n_max, void* cand,
                        float* out_scores = nullptr, const int32_t* id_offset = nullptr, int shift = 0) {
  const int nseg = seg_count(n_max, k, nq);
  if (nseg == 0)
    return launch_topk(src, v, scores, stride, q_seq, q_vis, pool, nq, k, out, out_stride, s, out_scores,
                       id_offset, shift);
  float* cs = static_cast<float*>(cand);
  int32_t* ci = reinterpret_cast<int32_t*>(cs + (int64_t)nq * nseg * k);
  cudaError_t e = launch_topk(src, v, scores, stride, q_seq, q_vis, pool, nq, k, ci, k, s, cs, id_offset, shift,
                              nseg);
  CacheView none{};
  if (e == cudaSuccess)
    e = launch_topk(kSrcCand, none, cs, (int64_t)nseg * k, nullptr, nullptr, ci, nq, k, out, out_stride, s,
                    out_scores);
  return e;
}

// Per-query floats of the indexer workspace: token (or block-key) scores, then,
// for a max-pooled Full call, the block maxima at offset nq * flat stride.
int64_t max_pool_block_stride(int64_t max_visible) {
  return ceil_div(ceil_div(max_visible, kBlock), kBlocksPerPage) * kBlocksPerPage;
}

size_t shard_attn_idx_offset(int nq, int heads) {
  return (attn_workspace_bytes(nq, heads) + 255) / 256 * 256;
}

int64_t indexer_stride(int64_t max_visible, int hierarchical);

// Segment candidates of an indexer call (the largest of its selections).
size_t indexer_seg_bytes(int nq, int64_t max_visible, int hierarchical) {
  const int64_t flat_n = ceil_div(max_visible, kBlock) * kBlock;
  const int64_t blocks_n = max_pool_block_stride(max_visible);
  size_t b = 0;
  if (hierarchical != CSA2_HIER_MEAN) b = seg_bytes(nq, flat_n, kTopK);                  // flat token top-k
  if (hierarchical != CSA2_HIER_FLAT) b = std::max(b, seg_bytes(nq, blocks_n, kPoolBlocks));  // block top-k
  return b;
}

int64_t indexer_stride(int64_t max_visible, int hierarchical) {
  const int64_t nb = ceil_div(max_visible, kBlock);
  if (hierarchical == CSA2_HIER_MAX) return nb * kBlock;
  if (hierarchical) {
    const int64_t bk = ceil_div(nb, kBlocksPerPage) * kBlocksPerPage;
    const int64_t pool = (int64_t)kPoolBlocks * kBlock;
    return bk > pool ? bk : pool;
  }
  return nb * kBlock;
}

}  // namespace

extern "C" {

void csa2_indexset_init(csa2_indexset* set, int32_t* idx, int32_t* pool_blocks, int32_t rows) {
  if (!set) return;
  set->idx = idx;
  set->pool_blocks = pool_blocks;
  set->rows = rows;
  set->layer = -1;
  set->mode = -1;
  set->pool_layer = -1;
  set->cache_id = 0;
  set->nq = 0;
  set->attn_rows = nullptr;
  set->rows_layer = -1;
  set->rows_split = 0;
  set->rows_nq = 0;
}

void csa2_indexset_attach_rows(csa2_indexset* set, int32_t* attn_rows) {
  if (!set) return;
  set->attn_rows = attn_rows;
  set->rows_layer = -1;
}

int csa2_kv_quant_append(const csa2_cache* cache, const uint16_t* kv, const uint16_t* idxk,
                         const int32_t* entry_seq, const int32_t* entry_pos, int32_t n,
                         int32_t compress, csa2_stream_t stream) {
  CacheView v;
  int st = make_view(cache, &v);
  if (st) return st;
  if (n < 0) return CSA2_ERR_INVALID_ARG;
  if (compress != 1 && compress != 2) return CSA2_ERR_SHAPE;
  if (n == 0) return CSA2_OK;
  if (!kv || !idxk || !entry_seq || !entry_pos) return CSA2_ERR_INVALID_ARG;
  if (!aligned(kv, 16) || !aligned(idxk, 4) || !aligned(entry_seq, 4) || !aligned(entry_pos, 4))
    return CSA2_ERR_ALIGNMENT;
  return from_cuda(launch_append(v, kv, idxk, entry_seq, entry_pos, n, compress, (cudaStream_t)stream));
}

int csa2_indexer_score_topk(const csa2_cache* cache, const uint16_t* idx_q, const float* head_w,
                            const int32_t* q_seq, const int32_t* q_visible, int32_t nq,
                            int64_t max_visible, int32_t mode, int32_t hierarchical, int32_t layer,
                            csa2_indexset* set, void* workspace, size_t workspace_bytes,
                            csa2_stream_t stream) {
  CacheView v;
  int st = make_view(cache, &v);
  if (st) return st;
  if (mode != CSA2_FULL && mode != CSA2_REINDEX) return CSA2_ERR_INVALID_ARG;
  if (nq < 0 || max_visible < 0 || max_visible > ((int64_t)1 << 31) - 1 || layer < 0)
    return CSA2_ERR_INVALID_ARG;
  if (!set || !set->idx) return CSA2_ERR_INVALID_ARG;
  if (hierarchical < CSA2_HIER_FLAT || hierarchical > CSA2_HIER_MAX) return CSA2_ERR_INVALID_ARG;
  if (nq > set->rows || nq > kMaxQueries) return CSA2_ERR_SHAPE;
  const bool hier = hierarchical != 0 || mode == CSA2_REINDEX;
  // the workspace layout this call uses (Reindex: pool scores)
  const int ws_kind = mode == CSA2_REINDEX ? CSA2_HIER_MEAN : hierarchical;
  if (hier && !set->pool_blocks) return CSA2_ERR_INVALID_ARG;
  if (mode == CSA2_REINDEX) {
    // Reindex ranks the pool of the last hierarchical Full layer on this cache
    if (set->pool_layer < 0 || set->pool_layer >= layer || set->cache_id != cache->cache_id ||
        nq > set->nq)
      return CSA2_ERR_MODE_STATE;
  }
  if (nq > 0 && (!idx_q || !q_seq)) return CSA2_ERR_INVALID_ARG;
  if (!aligned(idx_q, 16) || !aligned(head_w, 4) || !aligned(q_seq, 4) || !aligned(q_visible, 4) ||
      !aligned(set->idx, 4) || !aligned(set->pool_blocks, 4))
    return CSA2_ERR_ALIGNMENT;
  const size_t need = csa2_workspace_bytes(CSA2_OP_INDEXER, nq, 0, max_visible, ws_kind);
  if (nq > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16)))
    return CSA2_ERR_WORKSPACE;
  if (nq > 0) {
    if ((st = ensure_device_setup())) return st;
    cudaStream_t s = (cudaStream_t)stream;
    float* scores = static_cast<float*>(workspace);
    const int64_t stride = indexer_stride(max_visible, ws_kind);
    const int64_t nb = ceil_div(max_visible, kBlock);
    cudaError_t e = cudaSuccess;
    if (mode == CSA2_FULL && hierarchical == CSA2_HIER_MAX) {
      // every token scored once; the score kernel also writes each block's
      // maximum; the pool is the 2,048 best maxima, the tokens the flat top-512
      float* bmax = scores + (int64_t)nq * stride;
      const int64_t bstride = max_pool_block_stride(max_visible);
      void* cand = bmax + (int64_t)nq * bstride;
      e = launch_score(kSrcFlat, v, idx_q, head_w, q_seq, q_visible, nullptr, nq, nb, stride, scores,
                       bmax, bstride, s);
      if (e == cudaSuccess)
        e = select_topk(kSrcBlockKeys, v, bmax, bstride, q_seq, q_visible, nullptr, nq, kPoolBlocks,
                        set->pool_blocks, kPoolBlocks, s, bstride, cand);
      if (e == cudaSuccess)
        e = select_topk(kSrcFlat, v, scores, stride, q_seq, q_visible, nullptr, nq, kTopK, set->idx, kTopK, s,
                        nb * kBlock, cand);
    } else if (mode == CSA2_FULL && hier) {
      const int64_t bk_units = ceil_div(nb, kBlocksPerPage);
      e = launch_score(kSrcBlockKeys, v, idx_q, head_w, q_seq, q_visible, nullptr, nq, bk_units,
                       stride, scores, nullptr, 0, s);
      if (e == cudaSuccess)
        e = select_topk(kSrcBlockKeys, v, scores, stride, q_seq, q_visible, nullptr, nq, kPoolBlocks,
                        set->pool_blocks, kPoolBlocks, s, bk_units * kBlocksPerPage, scores + (int64_t)nq * stride);
    }
    if (e == cudaSuccess && hier && !(mode == CSA2_FULL && hierarchical == CSA2_HIER_MAX)) {
      e = launch_score(kSrcPool, v, idx_q, head_w, q_seq, q_visible, set->pool_blocks, nq,
                       kPoolBlocks, stride, scores, nullptr, 0, s);
      if (e == cudaSuccess)
        e = launch_topk(kSrcPool, v, scores, stride, q_seq, q_visible, set->pool_blocks, nq, kTopK,
                        set->idx, kTopK, s);
    }
    if (e == cudaSuccess && !hier) {
      e = launch_score(kSrcFlat, v, idx_q, head_w, q_seq, q_visible, nullptr, nq, nb, stride,
                       scores, nullptr, 0, s);
      if (e == cudaSuccess)
        e = select_topk(kSrcFlat, v, scores, stride, q_seq, q_visible, nullptr, nq, kTopK, set->idx, kTopK, s,
                        nb * kBlock, scores + (int64_t)nq * stride);
    }
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
  }
  set->layer = layer;
  set->mode = mode;
  set->cache_id = cache->cache_id;
  set->rows_layer = -1;   // the attention row cache belongs to the previous set
  if (mode == CSA2_FULL) {
    set->nq = nq;
    set->pool_layer = hier ? layer : -1;
  }
  return CSA2_OK;
}

int csa2_sparse_attn(const csa2_cache* cache, const uint16_t* q, int32_t heads, float sm_scale,
                     const int32_t* q_seq, const int32_t* q_visible, int32_t nq, int32_t mode,
                     int32_t layer, csa2_indexset* set, uint16_t* out, void* workspace,
                     size_t workspace_bytes, csa2_stream_t stream) {
  CacheView v;
  int st = make_view(cache, &v);
  if (st) return st;
  if (mode != CSA2_FULL && mode != CSA2_REINDEX && mode != CSA2_REUSE) return CSA2_ERR_INVALID_ARG;
  if (heads != 16 && heads != 32 && heads != 48 && heads != 64) return CSA2_ERR_SHAPE;
  if (nq < 0 || layer < 0 || !set || !set->idx) return CSA2_ERR_INVALID_ARG;
  if (nq > set->rows || nq > kMaxQueries) return CSA2_ERR_SHAPE;
  if (set->cache_id != cache->cache_id || set->layer < 0 || nq > set->nq) return CSA2_ERR_MODE_STATE;
  if (mode == CSA2_REUSE) {
    // Reuse consumes the latest Full / Reindex indices of an earlier layer
    if (set->layer >= layer || (set->mode != CSA2_FULL && set->mode != CSA2_REINDEX))
      return CSA2_ERR_MODE_STATE;
  } else if (set->layer != layer || set->mode != mode) {
    return CSA2_ERR_MODE_STATE;   // Full / Reindex attend over their own fresh set
  }
  if (nq > 0 && (!q || !q_seq || !out)) return CSA2_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(q_seq, 4) || !aligned(q_visible, 4))
    return CSA2_ERR_ALIGNMENT;
  const size_t need = csa2_workspace_bytes(CSA2_OP_ATTENTION, nq, heads, 0, 0);
  if (nq > 0 && need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16)))
    return CSA2_ERR_WORKSPACE;
  if (!aligned(set->attn_rows, 4)) return CSA2_ERR_ALIGNMENT;
  if (nq == 0) return CSA2_OK;
  if ((st = ensure_device_setup())) return st;
  // row cache: Full / Reindex record the resolved rows, Reuse reads them when they
  // come from the set's current indexer layer with the same queries and ranges
  const int split = attn_splits_for(nq);
  int rmode = 0;
  if (set->attn_rows) {
    if (mode != CSA2_REUSE) rmode = 1;
    else if (set->rows_layer == set->layer && set->rows_nq == nq && set->rows_split == split) rmode = 2;
  }
  const int e = from_cuda(launch_attention(v, q, heads, sm_scale, q_seq, q_visible, set->idx, nq, out,
                                           workspace, set->attn_rows, rmode, split, (cudaStream_t)stream));
  if (rmode == 1) {
    if (e == CSA2_OK) {
      set->rows_layer = layer;
      set->rows_nq = nq;
      set->rows_split = split;
    } else {
      set->rows_layer = -1;
    }
  }
  return e;
}

int csa2_swa_replay(const csa2_cache* cache, const uint16_t* kv_last, const uint16_t* idxk_last,
                    const uint8_t* miss, int32_t compress, csa2_stream_t stream) {
  CacheView v;
  int st = make_view(cache, &v);
  if (st) return st;
  if (compress != 1 && compress != 2) return CSA2_ERR_SHAPE;
  if (!kv_last || !miss || (!idxk_last && !v.swa)) return CSA2_ERR_INVALID_ARG;
  if (!aligned(kv_last, 16) || !aligned(idxk_last, 4)) return CSA2_ERR_ALIGNMENT;
  return from_cuda(launch_replay(v, kv_last, idxk_last, miss, compress, (cudaStream_t)stream));
}

size_t csa2_workspace_bytes(int32_t op, int32_t nq, int32_t heads, int64_t max_visible,
                            int32_t hierarchical) {
  if (nq < 0) return 0;
  if (op == CSA2_OP_INDEXER) {
    if (max_visible < 0) return 0;
    if (hierarchical < CSA2_HIER_FLAT || hierarchical > CSA2_HIER_MAX) return 0;
    int64_t per_query = indexer_stride(max_visible, hierarchical);
    if (hierarchical == CSA2_HIER_MAX) per_query += max_pool_block_stride(max_visible);
    return (size_t)nq * (size_t)per_query * sizeof(float) + indexer_seg_bytes(nq, max_visible, hierarchical) + 256;
  }
  if (op == CSA2_OP_ATTENTION) {
    if (heads != 16 && heads != 32 && heads != 48 && heads != 64) return 0;
    return attn_workspace_bytes(nq, heads);
  }
  if (op == CSA2_OP_SHARD_INDEXER) {   // scores, the local pool, segment candidates
    if (max_visible < 0) return 0;
    return (size_t)nq * (size_t)(indexer_stride(max_visible, CSA2_HIER_MEAN) + kPoolBlocks) * 4 +
           seg_bytes(nq, max_pool_block_stride(max_visible), kPoolBlocks) + 256;
  }
  if (op == CSA2_OP_SHARD_MERGE) {     // heads = shards, max_visible = candidates per shard
    if (heads < 1 || max_visible < 8 || max_visible % 8 != 0) return 0;
    return (size_t)nq * (size_t)heads * (size_t)max_visible * 8 + 256;
  }
  if (op == CSA2_OP_SHARD_ATTENTION) {  // attention slices, then local indices and window starts
    if (heads != 16 && heads != 32 && heads != 48 && heads != 64) return 0;
    return shard_attn_idx_offset(nq, heads) + (size_t)nq * (kTopK + 1) * 4 + 256;
  }
  return 0;
}

int csa2_shard_indexer_candidates(const csa2_cache* cache, const uint16_t* idx_q, const float* head_w,
                                  const int32_t* q_seq, const int32_t* shard_offset, int32_t nq,
                                  int64_t max_visible, int32_t stage, const int32_t* global_pool,
                                  float* cand_score, int32_t* cand_id, void* workspace,
                                  size_t workspace_bytes, csa2_stream_t stream) {
  CacheView v;
  int st = make_view(cache, &v);
  if (st) return st;
  if (stage != CSA2_SHARD_BLOCKS && stage != CSA2_SHARD_TOKENS) return CSA2_ERR_INVALID_ARG;
  if (nq < 0 || max_visible < 0 || max_visible > ((int64_t)1 << 31) - 1) return CSA2_ERR_INVALID_ARG;
  if (nq > kMaxQueries) return CSA2_ERR_SHAPE;
  if (nq == 0) return CSA2_OK;
  if (!idx_q || !q_seq || !shard_offset || !cand_score || !cand_id) return CSA2_ERR_INVALID_ARG;
  if (stage == CSA2_SHARD_TOKENS && !global_pool) return CSA2_ERR_INVALID_ARG;
  if (!aligned(idx_q, 16) || !aligned(head_w, 4) || !aligned(q_seq, 4) || !aligned(shard_offset, 4) ||
      !aligned(global_pool, 4) || !aligned(cand_score, 4) || !aligned(cand_id, 4))
    return CSA2_ERR_ALIGNMENT;
  const size_t need = csa2_workspace_bytes(CSA2_OP_SHARD_INDEXER, nq, 0, max_visible, 0);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return CSA2_ERR_WORKSPACE;
  if ((st = ensure_device_setup())) return st;
  cudaStream_t s = (cudaStream_t)stream;
  float* scores = static_cast<float*>(workspace);
  const int64_t stride = indexer_stride(max_visible, CSA2_HIER_MEAN);
  cudaError_t e;
  if (stage == CSA2_SHARD_BLOCKS) {
    const int64_t bk_units = ceil_div(ceil_div(max_visible, kBlock), kBlocksPerPage);
    e = launch_score(kSrcBlockKeys, v, idx_q, head_w, q_seq, nullptr, nullptr, nq, bk_units, stride, scores,
                     nullptr, 0, s);
    if (e == cudaSuccess)
      e = select_topk(kSrcBlockKeys, v, scores, stride, q_seq, nullptr, nullptr, nq, kPoolBlocks, cand_id,
                      kPoolBlocks, s, bk_units * kBlocksPerPage,
                      scores + (int64_t)nq * (stride + kPoolBlocks), cand_score, shard_offset, 3);
  } else {
    int32_t* lpool = reinterpret_cast<int32_t*>(scores + (int64_t)nq * stride);
    e = launch_shard_localize(v, q_seq, shard_offset, global_pool, kPoolBlocks, kBlock, lpool, nullptr, nullptr,
                              nq, s);
    if (e == cudaSuccess)
      e = launch_score(kSrcPool, v, idx_q, head_w, q_seq, nullptr, lpool, nq, kPoolBlocks, stride, scores,
                       nullptr, 0, s);
    if (e == cudaSuccess)
      e = launch_topk(kSrcPool, v, scores, stride, q_seq, nullptr, lpool, nq, kTopK, cand_id, kTopK, s,
                      cand_score, shard_offset, 0);
  }
  return from_cuda(e);
}

int csa2_shard_merge_topk(const float* cand_score, const int32_t* cand_id, int32_t nshard, int32_t nq,
                          int32_t n, int64_t query_stride, int64_t shard_stride, int32_t k,
                          int32_t* out_id, float* out_score, void* workspace, size_t workspace_bytes,
                          csa2_stream_t stream) {
  if (nshard < 1 || nq < 0 || n < 8 || n % 8 != 0 || k < 1 || query_stride < 0 || shard_stride < 0)
    return CSA2_ERR_INVALID_ARG;
  if (nq > kMaxQueries || (int64_t)nshard * n > ((int64_t)1 << 30)) return CSA2_ERR_SHAPE;
  if (nq == 0) return CSA2_OK;
  if (!cand_score || !cand_id || !out_id) return CSA2_ERR_INVALID_ARG;
  if (!aligned(cand_score, 4) || !aligned(cand_id, 4) || !aligned(out_id, 4) || !aligned(out_score, 4))
    return CSA2_ERR_ALIGNMENT;
  const size_t need = csa2_workspace_bytes(CSA2_OP_SHARD_MERGE, nq, nshard, n, 0);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return CSA2_ERR_WORKSPACE;
  int st;
  if ((st = ensure_device_setup())) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t m = (int64_t)nshard * n;
  float* pscore = static_cast<float*>(workspace);
  int32_t* pid = reinterpret_cast<int32_t*>(pscore + (int64_t)nq * m);
  cudaError_t e = launch_shard_pack(cand_score, cand_id, nshard, n, query_stride, shard_stride, nq, pscore, pid, s);
  CacheView none{};
  if (e == cudaSuccess)
    e = launch_topk(kSrcCand, none, pscore, m, nullptr, nullptr, pid, nq, k, out_id, k, s, out_score, nullptr, 0);
  return from_cuda(e);
}

int csa2_sparse_attn_shard(const csa2_cache* cache, const uint16_t* q, int32_t heads, float sm_scale,
                           const int32_t* q_seq, const int32_t* shard_offset, const int32_t* global_idx,
                           const int32_t* window_start, int32_t nq, uint16_t* out, float* lse2,
                           void* workspace, size_t workspace_bytes, csa2_stream_t stream) {
  CacheView v;
  int st = make_view(cache, &v);
  if (st) return st;
  if (heads != 16 && heads != 32 && heads != 48 && heads != 64) return CSA2_ERR_SHAPE;
  if (nq < 0) return CSA2_ERR_INVALID_ARG;
  if (nq > kMaxQueries) return CSA2_ERR_SHAPE;
  if (nq == 0) return CSA2_OK;
  if (!q || !q_seq || !shard_offset || !global_idx || !window_start || !out || !lse2) return CSA2_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(q_seq, 4) || !aligned(shard_offset, 4) ||
      !aligned(global_idx, 4) || !aligned(window_start, 4) || !aligned(lse2, 4))
    return CSA2_ERR_ALIGNMENT;
  const size_t need = csa2_workspace_bytes(CSA2_OP_SHARD_ATTENTION, nq, heads, 0, 0);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return CSA2_ERR_WORKSPACE;
  if ((st = ensure_device_setup())) return st;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t* lidx = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + shard_attn_idx_offset(nq, heads));
  int32_t* lwin = lidx + (int64_t)nq * kTopK;
  cudaError_t e = launch_shard_localize(v, q_seq, shard_offset, global_idx, kTopK, 1, lidx, window_start, lwin,
                                        nq, s);
  if (e == cudaSuccess)
    e = launch_attention(v, q, heads, sm_scale, q_seq, nullptr, lidx, nq, out, workspace, nullptr, 0,
                         attn_splits_for(nq), s, lwin, lse2);
  return from_cuda(e);
}

int csa2_shard_combine(const uint16_t* part, const float* lse2, int32_t nshard, int32_t nq, int32_t heads,
                       int64_t query_stride, int64_t shard_stride, uint16_t* out, csa2_stream_t stream) {
  if (nshard < 1 || nq < 0 || query_stride < 0 || shard_stride < 0) return CSA2_ERR_INVALID_ARG;
  if (heads != 16 && heads != 32 && heads != 48 && heads != 64) return CSA2_ERR_SHAPE;
  if (nq > kMaxQueries) return CSA2_ERR_SHAPE;
  if (nq == 0) return CSA2_OK;
  if (!part || !lse2 || !out) return CSA2_ERR_INVALID_ARG;
  if (!aligned(part, 16) || !aligned(out, 16) || !aligned(lse2, 4)) return CSA2_ERR_ALIGNMENT;
  return from_cuda(launch_shard_combine(part, lse2, nshard, nq, heads, query_stride, shard_stride, out,
                                        (cudaStream_t)stream));
}

int csa2_check_device_error(const csa2_cache* cache, csa2_stream_t stream, uint32_t* bits) {
  if (!cache || !cache->error_word) return CSA2_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t h = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return CSA2_ERR_CUDA;
  if (cudaMemcpyAsync(&h, cache->error_word, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return CSA2_ERR_CUDA;
  if (cudaMemsetAsync(cache->error_word, 0, sizeof(uint32_t), s) != cudaSuccess) return CSA2_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return CSA2_ERR_CUDA;
  if (bits) *bits = h;
  return h ? CSA2_ERR_DEVICE_BOUNDS : CSA2_OK;
}

const char* csa2_status_string(int status) {
  switch (status) {
    case CSA2_OK: return "ok";
    case CSA2_ERR_INVALID_ARG: return "invalid argument";
    case CSA2_ERR_SHAPE: return "unsupported shape";
    case CSA2_ERR_ALIGNMENT: return "misaligned pointer";
    case CSA2_ERR_MODE_STATE: return "layer mode called out of order";
    case CSA2_ERR_WORKSPACE: return "workspace missing or too small";
    case CSA2_ERR_CUDA: return "CUDA error";
    case CSA2_ERR_DEVICE_BOUNDS: return "kernel found an out-of-range page, position or sequence";
    default: return "unknown status";
  }
}

int csa2_version(void) { return 100; }

}  // extern "C"
