// Position-sharded decode of long sequences: each shard (one GPU's share of a
// sequence, a contiguous range of positions starting at a multiple of 8) runs
// the CSA2 step on its own positions, and three exchanges make the result the
// unsharded one:
//   1. every shard's 2,048 best blocks (score, global block id) are gathered
//      and merged into the global pool -- exact, since a block of the global
//      top-2048 is among its own shard's top-2048;
//   2. every shard ranks the pool's blocks that it holds, and the 512 best
//      (score, global position) of each are gathered and merged the same way;
//   3. every shard attends over the selected positions and the part of the
//      128-token window that it holds, and the partial outputs are merged by
//      their log-sum-exp (softmax over a union of disjoint sets).
// Candidate lists concatenated in shard order are in ascending global order,
// so a merge's "lowest position wins" tie-break is the unsharded one.
// (agentnet.co.il, "דיפסיק משיקה את V4.1-פלאש ...", section "CSA2: דחיסה
// לאורך ציר השכבות", for the pool, the 512 indices and the window.)
#include "common.cuh"

namespace csa2 {

// Global pool -> this shard's local pool (block ids of other shards -> -1), or
// global index set -> local positions (other shards' positions -> -1) and the
// window start in local positions.  One CTA per query.
__global__ void __launch_bounds__(256) shard_localize_kernel(CacheView c, const int32_t* __restrict__ q_seq,
                                                             const int32_t* __restrict__ shard_offset,
                                                             const int32_t* __restrict__ gin, int n, int unit,
                                                             int32_t* __restrict__ lout,
                                                             const int32_t* __restrict__ wstart_g,
                                                             int32_t* __restrict__ wstart_l) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  const int64_t off = shard_offset[r];
  const int64_t len = seq_len_of(c, q_seq[r]);
  // a shard with entries starts at a multiple of 8 (an empty one's offset is never used)
  if (threadIdx.x == 0 && len > 0 && (off < 0 || (off & (kBlock - 1)) != 0)) raise_error(c.err, CSA2_DEVERR_POS);
  const int64_t lo = off / unit, hi = (len + unit - 1) / unit;   // local ids [0, hi)
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int64_t g = gin[(int64_t)r * n + i];
    const int64_t l = g - lo;
    lout[(int64_t)r * n + i] = (g >= 0 && l >= 0 && l < hi) ? (int32_t)l : -1;
  }
  if (wstart_l != nullptr && threadIdx.x == 0) {
    const int64_t w = (int64_t)wstart_g[r] - off;
    wstart_l[r] = (int32_t)(w < 0 ? 0 : (w > len ? len : w));
  }
}

// Strided candidate lists (shard s of query q at row q qs + s ss, n entries
// each) -> contiguous rows of nshard n entries, shard-major within a row.
__global__ void shard_pack_kernel(const float* __restrict__ score, const int32_t* __restrict__ id, int nshard,
                                  int n, int64_t qs, int64_t ss, float* __restrict__ pscore,
                                  int32_t* __restrict__ pid) {
  pdl_wait();
  pdl_trigger();
  const int q = blockIdx.y;
  const int64_t m = (int64_t)nshard * n;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < m; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t s = i / n, j = i - s * n;
    const int64_t src = ((int64_t)q * qs + s * ss) * n + j;
    pscore[(int64_t)q * m + i] = score[src];
    pid[(int64_t)q * m + i] = id[src];
  }
}

// out[q][h] = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M), M = max_s lse_s,
// over the shards with a non-empty set; bf16 round to nearest even.  O_s are
// the shards' normalised outputs.  One CTA per (query, head), 4 channels per
// thread.
__global__ void __launch_bounds__(128) shard_combine_kernel(const uint16_t* __restrict__ part,
                                                            const float* __restrict__ lse2, int nshard, int H,
                                                            int64_t qs, int64_t ss, uint16_t* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int q = blockIdx.x, h = blockIdx.y;
  float M = -INFINITY;
  for (int s = 0; s < nshard; ++s) M = fmaxf(M, lse2[((int64_t)q * qs + s * ss) * H + h]);
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  float wsum = 0.0f;
  const int ch = 4 * threadIdx.x;
  if (M != -INFINITY) {
    for (int s = 0; s < nshard; ++s) {
      const int64_t row = (int64_t)q * qs + s * ss;
      const float l = lse2[row * H + h];
      if (l == -INFINITY) continue;
      const float wgt = exp2f(l - M);
      wsum += wgt;
      const uint2 v = *reinterpret_cast<const uint2*>(part + (row * H + h) * kD + ch);
      acc[0] = fmaf(wgt, bf16_lo(v.x), acc[0]);
      acc[1] = fmaf(wgt, bf16_hi(v.x), acc[1]);
      acc[2] = fmaf(wgt, bf16_lo(v.y), acc[2]);
      acc[3] = fmaf(wgt, bf16_hi(v.y), acc[3]);
    }
  }
  const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
  uint2 o;
  o.x = (uint32_t)f32_to_bf16_rne(acc[0] * inv) | ((uint32_t)f32_to_bf16_rne(acc[1] * inv) << 16);
  o.y = (uint32_t)f32_to_bf16_rne(acc[2] * inv) | ((uint32_t)f32_to_bf16_rne(acc[3] * inv) << 16);
  *reinterpret_cast<uint2*>(out + ((int64_t)q * H + h) * kD + ch) = o;
}

cudaError_t launch_shard_localize(const CacheView& c, const int32_t* q_seq, const int32_t* shard_offset,
                                  const int32_t* gin, int n, int unit, int32_t* lout, const int32_t* wstart_g,
                                  int32_t* wstart_l, int nq, cudaStream_t st) {
  if (nq == 0) return cudaSuccess;
  launch_pdl(shard_localize_kernel, nq, 256, 0, st, c, q_seq, shard_offset, gin, n, unit, lout, wstart_g, wstart_l);
  return cudaGetLastError();
}

cudaError_t launch_shard_pack(const float* score, const int32_t* id, int nshard, int n, int64_t qs, int64_t ss,
                              int nq, float* pscore, int32_t* pid, cudaStream_t st) {
  if (nq == 0) return cudaSuccess;
  const int64_t m = (int64_t)nshard * n;
  const int bx = (int)((m + 255) / 256 < 64 ? (m + 255) / 256 : 64);
  launch_pdl(shard_pack_kernel, dim3(bx, nq), 256, 0, st, score, id, nshard, n, qs, ss, pscore, pid);
  return cudaGetLastError();
}

cudaError_t launch_shard_combine(const uint16_t* part, const float* lse2, int nshard, int nq, int H, int64_t qs,
                                 int64_t ss, uint16_t* out, cudaStream_t st) {
  if (nq == 0) return cudaSuccess;
  launch_pdl(shard_combine_kernel, dim3(nq, H), kD / 4, 0, st, part, lse2, nshard, H, qs, ss, out);
  return cudaGetLastError();
}

}  // namespace csa2
