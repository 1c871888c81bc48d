// Definitions shared by the indexer kernels: candidate-unit sources and the
// per-query unit counts.
#pragma once

#include "common.cuh"

namespace csa2 {

// SRC_CAND (top-k only): explicit candidates -- scores[r][i] with the id of
// entry i in cand_ids[r][i], the entries of a row in ascending id order.
enum UnitSource : int { SRC_FLAT = 0, SRC_BLOCKKEYS = 1, SRC_POOL = 2, SRC_CAND = 3 };

__device__ __forceinline__ int64_t visible_of(const CacheView& c, const int32_t* q_seq,
                                              const int32_t* q_vis, int r) {
  return q_vis ? (int64_t)q_vis[r] : (int64_t)seq_len_of(c, q_seq[r]);
}

// Number of units of query r for a source.
__device__ __forceinline__ int64_t units_of(int src, int64_t v) {
  const int64_t nb = (v + kBlock - 1) / kBlock;
  if (src == SRC_FLAT) return nb;
  if (src == SRC_BLOCKKEYS) return (nb + kBlocksPerPage - 1) / kBlocksPerPage;
  return kPoolBlocks;
}

}  // namespace csa2
