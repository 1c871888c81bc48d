// CSA2 indexer: score streaming over 1-KiB key units + exact radix top-k.
//
// The indexer of a Full layer picks 512 fresh indices; a Reindex layer ranks
// the last Full layer's indexer K with its own indexer Q; in the decoder the
// Full layer first narrows the context to a pool of 2,048 blocks x 8 tokens
// (agentnet.co.il, "דיפסיק משיקה את V4.1-פלאש ...", section "CSA2: דחיסה
// לאורך ציר השכבות").  Every candidate set here is made of 1-KiB units of
// eight 128-B bf16 key rows that are contiguous in HBM:
//   FLAT      unit u = tokens 8u..8u+7 of the indexer-key pages,
//   BLOCKKEYS unit u = the 8 block keys stored in page slot u,
//   POOL      unit u = the 8 tokens of pool block pool[u].
// score(q, k) = sum_h w_h * max(0, q_h . k), fp32.
//
// Scoring is HBM-bound (4 heads x 64 dims = 4 FLOP per key byte): each warp
// streams whole units with 16-B non-allocating loads, several units in flight
// per lane; lane l holds 16 dims of row l/4, so a row's four partial dot
// products meet in two shuffles.  Scores go to the caller's workspace (4 B
// per 128-B key) and a second kernel selects the top k.
//
// Top-k: one CTA per query.  Keys are the order-preserving uint32 image of
// the scores (-inf, the "not a candidate" marker, maps to 0).  A 12/12/8-bit
// radix select finds the k-th largest key T and how many entries equal to T
// are needed; a final pass in position order keeps every key > T and the
// lowest-position entries equal to T, so the tie-break is "lowest position
// wins" and the output comes out in ascending position order.
#include "common.cuh"

namespace csa2 {

enum UnitSource : int { SRC_FLAT = 0, SRC_BLOCKKEYS = 1, SRC_POOL = 2 };

constexpr int kScoreWarps = 8;
constexpr int kUnitsPerWarp = 4;
constexpr int kUnitsPerCta = kScoreWarps * kUnitsPerWarp;  // 32

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

template <int SRC>
__global__ void __launch_bounds__(256) score_units_kernel(CacheView c, const uint16_t* __restrict__ idx_q,
                                                          const float* __restrict__ head_w,
                                                          const int32_t* __restrict__ q_seq,
                                                          const int32_t* __restrict__ q_vis,
                                                          const int32_t* __restrict__ pool,
                                                          int64_t max_units, int64_t stride,
                                                          float* __restrict__ scores) {
  const int r = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int seq = q_seq[r];
  const int64_t v = visible_of(c, q_seq, q_vis, r);
  int64_t nunits = units_of(SRC, v);
  if (nunits > max_units) {   // visible length beyond the bound the call was sized for
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(c.err, CSA2_DEVERR_POS);
    nunits = max_units;
  }
  const int64_t u0 = (int64_t)blockIdx.x * kUnitsPerCta + warp * kUnitsPerWarp;
  if (u0 >= nunits) return;
  const int64_t nb = (v + kBlock - 1) / kBlock;

  // this lane's 16 dims of each head's query
  const int row = lane >> 2;
  const int dq = (lane & 3) * 16;
  float q[kIdxHeads][16];
#pragma unroll
  for (int h = 0; h < kIdxHeads; ++h) {
    const uint4* qp = reinterpret_cast<const uint4*>(idx_q + ((int64_t)r * kIdxHeads + h) * kIdxDim + dq);
    const uint4 a = __ldg(qp), b = __ldg(qp + 1);
    q[h][0] = bf16_lo(a.x); q[h][1] = bf16_hi(a.x); q[h][2] = bf16_lo(a.y); q[h][3] = bf16_hi(a.y);
    q[h][4] = bf16_lo(a.z); q[h][5] = bf16_hi(a.z); q[h][6] = bf16_lo(a.w); q[h][7] = bf16_hi(a.w);
    q[h][8] = bf16_lo(b.x); q[h][9] = bf16_hi(b.x); q[h][10] = bf16_lo(b.y); q[h][11] = bf16_hi(b.y);
    q[h][12] = bf16_lo(b.z); q[h][13] = bf16_hi(b.z); q[h][14] = bf16_lo(b.w); q[h][15] = bf16_hi(b.w);
  }
  float w[kIdxHeads];
#pragma unroll
  for (int h = 0; h < kIdxHeads; ++h) w[h] = head_w ? __ldg(head_w + (int64_t)r * kIdxHeads + h) : 1.0f;

  // issue every unit's loads first, then compute
  uint4 ka[kUnitsPerWarp], kb[kUnitsPerWarp];
  bool ok[kUnitsPerWarp];
#pragma unroll
  for (int i = 0; i < kUnitsPerWarp; ++i) {
    const int64_t u = u0 + i;
    const uint8_t* base = nullptr;
    ok[i] = false;
    if (u < nunits) {
      if (SRC == SRC_FLAT) {
        const int64_t pg = page_of(c, seq, u * kBlock);
        if (pg >= 0) {
          base = c.idxk + pg * kIdxPageBytes + (u & (kBlocksPerPage - 1)) * (kBlock * kIdxRowBytes);
          ok[i] = (u * kBlock + row) < v;
        }
      } else if (SRC == SRC_BLOCKKEYS) {
        const int64_t pg = page_of(c, seq, u * kPageTokens);
        if (pg >= 0) {
          base = c.bk + pg * kBkPageBytes;
          ok[i] = (u * kBlocksPerPage + row) < nb;
        }
      } else {
        const int32_t blk = pool[(int64_t)r * kPoolBlocks + u];
        if (blk >= 0) {
          if ((int64_t)blk >= nb) {
            raise_error(c.err, CSA2_DEVERR_POS);
          } else {
            const int64_t pg = page_of(c, seq, (int64_t)blk * kBlock);
            if (pg >= 0) {
              base = c.idxk + pg * kIdxPageBytes + (blk & (kBlocksPerPage - 1)) * (kBlock * kIdxRowBytes);
              ok[i] = ((int64_t)blk * kBlock + row) < v;
            }
          }
        }
      }
    }
    if (base != nullptr) {
      const uint8_t* p = base + row * kIdxRowBytes + dq * 2;
      ka[i] = ld_stream16(p);
      kb[i] = ld_stream16(p + 16);
    } else {
      ka[i] = make_uint4(0, 0, 0, 0);
      kb[i] = ka[i];
    }
  }
#pragma unroll
  for (int i = 0; i < kUnitsPerWarp; ++i) {
    const int64_t u = u0 + i;
    float k[16];
    k[0] = bf16_lo(ka[i].x); k[1] = bf16_hi(ka[i].x); k[2] = bf16_lo(ka[i].y); k[3] = bf16_hi(ka[i].y);
    k[4] = bf16_lo(ka[i].z); k[5] = bf16_hi(ka[i].z); k[6] = bf16_lo(ka[i].w); k[7] = bf16_hi(ka[i].w);
    k[8] = bf16_lo(kb[i].x); k[9] = bf16_hi(kb[i].x); k[10] = bf16_lo(kb[i].y); k[11] = bf16_hi(kb[i].y);
    k[12] = bf16_lo(kb[i].z); k[13] = bf16_hi(kb[i].z); k[14] = bf16_lo(kb[i].w); k[15] = bf16_hi(kb[i].w);
    float s = 0.0f;
#pragma unroll
    for (int h = 0; h < kIdxHeads; ++h) {
      float p = 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) p = fmaf(q[h][j], k[j], p);
      p += __shfl_xor_sync(0xffffffffu, p, 1);
      p += __shfl_xor_sync(0xffffffffu, p, 2);
      s = fmaf(w[h], fmaxf(p, 0.0f), s);
    }
    if (u < nunits && (lane & 3) == 0) {
      scores[(int64_t)r * stride + u * kBlock + row] = ok[i] ? s : -INFINITY;
    }
  }
}

// ---------------------------------------------------------------------------
// top-k
// ---------------------------------------------------------------------------

constexpr int kTopkThreads = 1024;
constexpr int kTopkSmemKeys = 16384;   // keys cached in shared memory up to this count

// Exclusive scan of one value per thread across the CTA (1024 threads).
// Returns the exclusive prefix; *total receives the CTA-wide sum.
__device__ __forceinline__ uint32_t cta_exclusive_scan(uint32_t v, uint32_t* warp_sums, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t s = warp_sums[lane];
    uint32_t t = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_sums[lane] = t - s;   // exclusive prefix of warp sums
    if (lane == 31) warp_sums[32] = t;
  }
  __syncthreads();
  const uint32_t res = warp_sums[warp] + x - v;
  *total = warp_sums[32];
  __syncthreads();
  return res;
}

struct TopkSmem {
  uint32_t hist[4096];
  uint32_t warp_sums[33];
  uint32_t bucket, above;   // result of a bucket search
  uint32_t nvalid;
};

// Find the bucket holding the k_rem-th largest element of a histogram of
// `nbins` bins (bins ordered by key; larger bin = larger key).  Sets
// sm->bucket and sm->above (elements in higher bins).
__device__ __forceinline__ void find_bucket(TopkSmem* sm, int nbins, uint32_t k_rem) {
  // thread t owns bins [nbins - 4(t+1), nbins - 4t) counted from the top
  const int per = 4;
  const int t = threadIdx.x;
  uint32_t local = 0;
  const int hi = nbins - per * t;   // exclusive upper bin
  if (hi > 0) {
#pragma unroll
    for (int j = 1; j <= per; ++j)
      if (hi - j >= 0) local += sm->hist[hi - j];
  }
  uint32_t total;
  const uint32_t before = cta_exclusive_scan(local, sm->warp_sums, &total);
  if (hi > 0 && before < k_rem && before + local >= k_rem) {
    uint32_t cum = before;
    for (int j = 1; j <= per; ++j) {
      const int b = hi - j;
      if (b < 0) break;
      const uint32_t hcount = sm->hist[b];
      if (cum + hcount >= k_rem) {
        sm->bucket = (uint32_t)b;
        sm->above = cum;
        break;
      }
      cum += hcount;
    }
  }
  __syncthreads();
}

template <int SRC>
__device__ __forceinline__ int32_t map_out(int64_t i, const int32_t* pool_row) {
  if (SRC == SRC_POOL) return pool_row[i >> 3] * kBlock + (int32_t)(i & 7);
  return (int32_t)i;
}

// One CTA per query: select the k best entries of scores[r][0 .. n_r).
template <int SRC>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(CacheView c, const float* __restrict__ scores,
                                                            int64_t stride, const int32_t* __restrict__ q_seq,
                                                            const int32_t* __restrict__ q_vis,
                                                            const int32_t* __restrict__ pool, int k,
                                                            int32_t* __restrict__ out, int64_t out_stride) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem* sm = reinterpret_cast<TopkSmem*>(smem_raw);
  uint32_t* keys_sm = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkSmem));

  const int r = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t v = visible_of(c, q_seq, q_vis, r);
  const int64_t n = min(units_of(SRC, v) * kBlock, stride);
  const float* srow = scores + (int64_t)r * stride;
  const int32_t* pool_row = pool ? pool + (int64_t)r * kPoolBlocks : nullptr;
  int32_t* orow = out + (int64_t)r * out_stride;
  const bool cached = n <= kTopkSmemKeys;

  // pass 0: keys (cached), valid count, 12-bit histogram of the top digit
  for (int i = tid; i < 4096; i += kTopkThreads) sm->hist[i] = 0;
  if (tid == 0) sm->nvalid = 0;
  __syncthreads();
  uint32_t myvalid = 0;
  for (int64_t i = tid; i < n; i += kTopkThreads) {
    const uint32_t key = score_key(srow[i]);
    if (cached) keys_sm[i] = key;
    if (key) {
      ++myvalid;
      atomicAdd(&sm->hist[key >> 20], 1u);
    }
  }
  atomicAdd(&sm->nvalid, myvalid);
  __syncthreads();
  const uint32_t nvalid = sm->nvalid;
  auto key_at = [&](int64_t i) -> uint32_t { return cached ? keys_sm[i] : score_key(srow[i]); };

  uint32_t T = 1u;           // select keys >= T ... refined below
  uint32_t need_eq = 0xFFFFFFFFu;
  if (nvalid > (uint32_t)k) {
    uint32_t k_rem = (uint32_t)k;
    find_bucket(sm, 4096, k_rem);
    uint32_t prefix = sm->bucket << 20;
    k_rem -= sm->above;
    // pass 1: bits 19..8 among keys with the same top 12 bits
    for (int i = tid; i < 4096; i += kTopkThreads) sm->hist[i] = 0;
    __syncthreads();
    for (int64_t i = tid; i < n; i += kTopkThreads) {
      const uint32_t key = key_at(i);
      if ((key & 0xFFF00000u) == prefix) atomicAdd(&sm->hist[(key >> 8) & 0xFFFu], 1u);
    }
    __syncthreads();
    find_bucket(sm, 4096, k_rem);
    prefix |= sm->bucket << 8;
    k_rem -= sm->above;
    // pass 2: bits 7..0
    for (int i = tid; i < 256; i += kTopkThreads) sm->hist[i] = 0;
    __syncthreads();
    for (int64_t i = tid; i < n; i += kTopkThreads) {
      const uint32_t key = key_at(i);
      if ((key & 0xFFFFFF00u) == prefix) atomicAdd(&sm->hist[key & 0xFFu], 1u);
    }
    __syncthreads();
    find_bucket(sm, 256, k_rem);
    T = prefix | sm->bucket;
    k_rem -= sm->above;
    need_eq = k_rem;          // how many entries equal to T to keep (lowest positions)
  }

  // final pass in position order: keep key > T, and key == T while need_eq lasts
  uint32_t base_sel = 0, base_eq = 0;
  for (int64_t c0 = 0; c0 < n; c0 += kTopkThreads) {
    const int64_t i = c0 + tid;
    uint32_t key = 0;
    if (i < n) key = key_at(i);
    const uint32_t gt = (key != 0 && key > T) ? 1u : 0u;
    const uint32_t eq = (key != 0 && key == T) ? 1u : 0u;
    uint32_t tot_eq;
    const uint32_t eq_rank = cta_exclusive_scan(eq, sm->warp_sums, &tot_eq) + base_eq;
    const uint32_t sel = gt | ((eq && eq_rank < need_eq) ? 1u : 0u);
    uint32_t tot_sel;
    const uint32_t slot = cta_exclusive_scan(sel, sm->warp_sums, &tot_sel) + base_sel;
    if (sel && slot < (uint32_t)k) orow[slot] = map_out<SRC>(i, pool_row);
    base_sel += tot_sel;
    base_eq += tot_eq;
    if (base_sel >= (uint32_t)k) break;
  }
  for (int64_t s = (int64_t)base_sel + tid; s < k; s += kTopkThreads) orow[s] = -1;
}

}  // namespace csa2

// ---- launchers used by api.cu ----
namespace csa2 {

size_t topk_smem_bytes() { return sizeof(TopkSmem) + (size_t)kTopkSmemKeys * 4; }

// Opt the top-k kernels in to their shared-memory size (once per device).
cudaError_t indexer_set_attributes() {
  const int smem = (int)topk_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(topk_kernel<SRC_FLAT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(topk_kernel<SRC_BLOCKKEYS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(topk_kernel<SRC_POOL>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return e;
}

// Scores of every query's units into `scores` (row stride `stride` floats).
cudaError_t launch_score(int src, const CacheView& c, const uint16_t* idx_q, const float* head_w,
                         const int32_t* q_seq, const int32_t* q_vis, const int32_t* pool, int nq,
                         int64_t max_units, int64_t stride, float* scores, cudaStream_t st) {
  dim3 grid((unsigned)((max_units + kUnitsPerCta - 1) / kUnitsPerCta), (unsigned)nq);
  if (grid.x == 0) return cudaSuccess;
  if (src == SRC_FLAT)
    score_units_kernel<SRC_FLAT><<<grid, 256, 0, st>>>(c, idx_q, head_w, q_seq, q_vis, pool, max_units, stride, scores);
  else if (src == SRC_BLOCKKEYS)
    score_units_kernel<SRC_BLOCKKEYS><<<grid, 256, 0, st>>>(c, idx_q, head_w, q_seq, q_vis, pool, max_units, stride, scores);
  else
    score_units_kernel<SRC_POOL><<<grid, 256, 0, st>>>(c, idx_q, head_w, q_seq, q_vis, pool, max_units, stride, scores);
  return cudaGetLastError();
}

cudaError_t launch_topk(int src, const CacheView& c, const float* scores, int64_t stride,
                        const int32_t* q_seq, const int32_t* q_vis, const int32_t* pool, int nq,
                        int k, int32_t* out, int64_t out_stride, cudaStream_t st) {
  const size_t smem = topk_smem_bytes();
  if (nq == 0) return cudaSuccess;
  if (src == SRC_FLAT)
    topk_kernel<SRC_FLAT><<<nq, kTopkThreads, smem, st>>>(c, scores, stride, q_seq, q_vis, pool, k, out, out_stride);
  else if (src == SRC_BLOCKKEYS)
    topk_kernel<SRC_BLOCKKEYS><<<nq, kTopkThreads, smem, st>>>(c, scores, stride, q_seq, q_vis, pool, k, out, out_stride);
  else
    topk_kernel<SRC_POOL><<<nq, kTopkThreads, smem, st>>>(c, scores, stride, q_seq, q_vis, pool, k, out, out_stride);
  return cudaGetLastError();
}

}  // namespace csa2
