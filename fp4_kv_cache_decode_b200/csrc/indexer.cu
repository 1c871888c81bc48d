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
// FP8 indexer keys (E4M3 codes + one fp32 scale s per token): a unit is the 8
// tokens' 512 code bytes plus their 32 scale bytes, and a key scores
// s x score(q, code values) -- s >= 0 commutes with the ReLU.
//
// Scoring of bf16 keys runs on the tensor cores (score_mma.cu).  The kernel
// here scores FP8 keys on the FMA pipes: each warp streams whole units through
// a cp.async ring, lane l holds 16 dims of row l/4 (E4M3 pairs converted to
// fp32), so a row's four partial dot products meet in two shuffles.  Scores go
// to the caller's workspace (4 B per key) and a second kernel selects the top k.
//
// Top-k: one CTA per query.  Keys are the order-preserving uint32 image of
// the scores (-inf, the "not a candidate" marker, maps to 0).  A 12/12/8-bit
// radix select finds the k-th largest key T and how many entries equal to T
// are needed; a final pass in position order keeps every key > T and the
// lowest-position entries equal to T, so the tie-break is "lowest position
// wins" and the output comes out in ascending position order.
#include "common.cuh"
#include "indexer.cuh"

namespace csa2 {

// Where a top-k writes: ids [nq][stride] (-1 padded), optionally the selected
// scores (same layout, -inf padded), and optionally a per-query offset added to
// every selected id, id_offset[r] >> offset_shift (a shard's first global
// position, or its first block with shift 3).
struct TopkOut {
  int32_t* ids;
  int64_t stride;
  float* scores;
  const int32_t* id_offset;
  int offset_shift;
  int nseg;   // > 1: CTA b takes segment b % nseg (seg_len entries) of row b / nseg and
              // writes its own output row b (ids offset by the segment's start)
  int seg_len;
};

// Inverse of score_key on non-zero keys (exact; -0 comes back as +0).
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / 32;
constexpr int kUnitsPerCta = 256;                         // at most 256 KiB of keys per CTA
constexpr int kStages = 3;

// Pipeline geometry per key format: 32 units per stage of 1 KiB (bf16 keys) or
// 544 B (FP8 codes + scales).  The scoring is bound by issue latency, not by
// the bytes in flight: 64-unit FP8 stages (the same bytes per stage as bf16)
// were measured slower.
template <bool F8>
struct ScoreGeom {
  static constexpr int kUnits = 32;                           // units per stage
  static constexpr int kWarpUnits = kUnits / kScoreWarps;     // per warp per stage
  static constexpr uint32_t kSlot = F8 ? 544u : 1024u;        // bytes per unit slot
  static constexpr uint32_t kSmem = kStages * kUnits * kSlot;
};
constexpr uint32_t kScoreSmemMax = ScoreGeom<false>::kSmem;   // 98,304 B
static_assert(ScoreGeom<true>::kSmem <= kScoreSmemMax, "stage sizes");

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// One CTA scores up to 256 consecutive units of one query:
//  1. thread t resolves unit t's HBM address (pool entry, page table) and how
//     many of its 8 rows are candidates -- all 256 lookups in flight at once;
//  2. the units stream through a 3-stage ring of 32-KiB shared-memory stages
//     with cp.async (lane l of a warp copies bytes 32l..32l+31 of each of the
//     warp's 4 units per stage), two stages ahead of the compute;
//  3. each lane reads back exactly the bytes it copied (row l/4, dims
//     16(l%4)..+15), forms its 4 partial head dot products, and two shuffles
//     finish each row's dot products.  No CTA-wide barrier inside the stream.
template <int SRC, bool F8>
__global__ void __launch_bounds__(kScoreThreads, 2) score_units_kernel(CacheView c, const uint16_t* __restrict__ idx_q,
                                                                       const float* __restrict__ head_w,
                                                                       const int32_t* __restrict__ q_seq,
                                                                       const int32_t* __restrict__ q_vis,
                                                                       const int32_t* __restrict__ pool,
                                                                       int64_t max_units, int64_t stride,
                                                                       int upc, float* __restrict__ scores,
                                                                       float* __restrict__ block_max,
                                                                       int64_t bstride) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t stage[];
  static_assert(!F8 || SRC != SRC_BLOCKKEYS, "block keys are bf16");
  __shared__ const uint8_t* ubase[kUnitsPerCta];
  __shared__ const uint8_t* uscale[F8 ? kUnitsPerCta : 1];   // FP8: the unit's 8 scales
  __shared__ int32_t urows[kUnitsPerCta];
  const int r = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int seq = q_seq[r];
  const int64_t v = visible_of(c, q_seq, q_vis, r);
  int64_t nunits = units_of(SRC, v);
  if (nunits > max_units) {   // visible length beyond the bound the call was sized for
    if (blockIdx.x == 0 && tid == 0) raise_error(c.err, CSA2_DEVERR_POS);
    nunits = max_units;
  }
  using G = ScoreGeom<F8>;
  const int64_t u0 = (int64_t)blockIdx.x * upc;   // upc <= kUnitsPerCta, a multiple of G::kUnits
  if (u0 >= nunits) return;
  const int64_t nb = (v + kBlock - 1) / kBlock;
  const int nu = (int)(nunits - u0 < upc ? nunits - u0 : upc);

  // 1. unit addresses and candidate rows
  {
    const int64_t u = u0 + tid;
    const uint8_t* base = nullptr;
    const uint8_t* sbase = nullptr;
    int nrows = 0;
    // the unit's codes (and, FP8, scales) within an indexer-key page
    auto unit_at = [&](int64_t pg, int64_t slot8) {
      if (F8) {
        base = c.idxk + pg * kIdx8PageBytes + slot8 * (kBlock * kIdx8RowBytes);
        sbase = c.idxk + pg * kIdx8PageBytes + kIdx8ScaleOff + slot8 * (kBlock * 4);
      } else {
        base = c.idxk + pg * kIdxPageBytes + slot8 * (kBlock * kIdxRowBytes);
      }
    };
    if (tid < nu) {
      if (SRC == SRC_FLAT) {
        const int64_t pg = page_of(c, seq, u * kBlock);
        if (pg >= 0) {
          unit_at(pg, u & (kBlocksPerPage - 1));
          nrows = (int)(v - u * kBlock < kBlock ? v - u * kBlock : kBlock);
        }
      } else if (SRC == SRC_BLOCKKEYS) {
        const int64_t pg = page_of(c, seq, u * kPageTokens);
        if (pg >= 0) {
          base = c.bk + pg * kBkPageBytes;
          nrows = (int)(nb - u * kBlocksPerPage < kBlocksPerPage ? nb - u * kBlocksPerPage : kBlocksPerPage);
        }
      } else {
        const int32_t blk = pool[(int64_t)r * kPoolBlocks + u];
        if (blk >= 0) {
          if ((int64_t)blk >= nb) {
            raise_error(c.err, CSA2_DEVERR_POS);
          } else {
            const int64_t pg = page_of(c, seq, (int64_t)blk * kBlock);
            if (pg >= 0) {
              unit_at(pg, blk & (kBlocksPerPage - 1));
              nrows = (int)(v - (int64_t)blk * kBlock < kBlock ? v - (int64_t)blk * kBlock : kBlock);
            }
          }
        }
      }
    }
    ubase[tid] = base;
    if (F8) uscale[F8 ? tid : 0] = sbase;
    urows[tid] = nrows;
  }

  // this lane's 16 dims of each head's query as 8 (even, odd) pairs (loaded while
  // the lookups run); the lane's head after the reduce-scatter below is hsel
  const int row = lane >> 2;
  const int dq = (lane & 3) * 16;
  float2 q[kIdxHeads][8];
#pragma unroll
  for (int h = 0; h < kIdxHeads; ++h) {
    const uint4* qp = reinterpret_cast<const uint4*>(idx_q + ((int64_t)r * kIdxHeads + h) * kIdxDim + dq);
    const uint4 a = __ldg(qp), b = __ldg(qp + 1);
    const uint32_t wq[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) q[h][j] = make_float2(bf16_lo(wq[j]), bf16_hi(wq[j]));
  }
  const int hsel = ((lane & 1) << 1) | ((lane >> 1) & 1);
  const float wsel = head_w ? __ldg(head_w + (int64_t)r * kIdxHeads + hsel) : 1.0f;
  __syncthreads();

  const uint32_t stage_s = (uint32_t)__cvta_generic_to_shared(stage);
  const int nstage = (nu + G::kUnits - 1) / G::kUnits;
  // issue the copies of stage s (this warp's units) into ring slot s % kStages
  auto issue = [&](int st) {
    if (st < nstage) {
#pragma unroll
      for (int i = 0; i < G::kWarpUnits; ++i) {
        const int j = st * G::kUnits + warp * G::kWarpUnits + i;
        const uint8_t* base = ubase[j];
        const uint32_t dst = stage_s + ((st % kStages) * G::kUnits + warp * G::kWarpUnits + i) * G::kSlot;
        if (j < nu && base != nullptr) {
          if (F8) {   // 512 code bytes, then the 32 scale bytes
            cp_async16(dst + lane * 16u, base + lane * 16);
            if (lane < 2) cp_async16(dst + 512u + lane * 16u, uscale[F8 ? j : 0] + lane * 16);
          } else {
            cp_async16(dst + lane * 32u, base + lane * 32);
            cp_async16(dst + lane * 32u + 16u, base + lane * 32 + 16);
          }
        }
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  issue(0);
  issue(1);
#pragma unroll 1
  for (int st = 0; st < nstage; ++st) {
    issue(st + 2);
    asm volatile("cp.async.wait_group 2;" ::: "memory");
#pragma unroll
    for (int i = 0; i < G::kWarpUnits; ++i) {
      const int j = st * G::kUnits + warp * G::kWarpUnits + i;
      const int64_t u = u0 + j;
      const bool have = j < nu && ubase[j] != nullptr;
      const uint8_t* su = stage + ((st % kStages) * G::kUnits + warp * G::kWarpUnits + i) * G::kSlot;
      float2 k[8];
      float srow = 1.0f;   // FP8: the row's scale
      if (F8) {            // lane l: code bytes 16l..16l+15 = row l/4, dims 16(l%4)..
        uint4 kc = make_uint4(0, 0, 0, 0);
        if (have) {
          kc = *reinterpret_cast<const uint4*>(su + lane * 16);
          srow = *reinterpret_cast<const float*>(su + 512 + row * 4);
        }
        const uint32_t wc[4] = {kc.x, kc.y, kc.z, kc.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) k[j] = e4m3x2_to_float2(wc[j >> 1] >> (16 * (j & 1)));
      } else {
        uint4 ka = make_uint4(0, 0, 0, 0), kb = ka;
        if (have) {
          ka = *reinterpret_cast<const uint4*>(su + lane * 32);
          kb = *reinterpret_cast<const uint4*>(su + lane * 32 + 16);
        }
        const uint32_t wk[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) k[j] = make_float2(bf16_lo(wk[j]), bf16_hi(wk[j]));
      }
      // partial dot products of the lane's 16 dims, even and odd dims in the two halves
      float p[kIdxHeads];
#pragma unroll
      for (int h = 0; h < kIdxHeads; ++h) {
        float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc = __ffma2_rn(q[h][j], k[j], acc);
        p[h] = acc.x + acc.y;
      }
      // the row's 4 lanes reduce-scatter the 4 heads: lane bit 0 keeps heads
      // {0,1} or {2,3}, lane bit 1 then keeps one of the pair (head hsel)
      {
        const bool b0 = (lane & 1) != 0;
        const float s0 = __shfl_xor_sync(0xffffffffu, b0 ? p[0] : p[2], 1);
        const float s1 = __shfl_xor_sync(0xffffffffu, b0 ? p[1] : p[3], 1);
        const float k0 = (b0 ? p[2] : p[0]) + s0, k1 = (b0 ? p[3] : p[1]) + s1;
        const bool b1 = (lane & 2) != 0;
        const float t0 = __shfl_xor_sync(0xffffffffu, b1 ? k0 : k1, 2);
        p[0] = (b1 ? k1 : k0) + t0;
      }
      float sc = wsel * fmaxf(p[0], 0.0f);
      sc += __shfl_xor_sync(0xffffffffu, sc, 1);
      sc += __shfl_xor_sync(0xffffffffu, sc, 2);
      if (F8) sc *= srow;
      const float val = row < urows[j] ? sc : -INFINITY;
      if (j < nu && (lane & 3) == 0) scores[(int64_t)r * stride + u * kBlock + row] = val;
      if (SRC == SRC_FLAT && block_max != nullptr) {   // max-pooled block score of block u
        float m = fmaxf(val, __shfl_xor_sync(0xffffffffu, val, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        float* brow = block_max + (int64_t)r * bstride;
        if (j < nu && lane == 0) brow[u] = m;
        // the last block's CTA pads the row to a whole 8-block unit with -inf
        if (j < nu && u == nunits - 1 && lane < kBlocksPerPage) {
          const int64_t pad = nunits + lane;
          if (pad < (nunits + kBlocksPerPage - 1) / kBlocksPerPage * kBlocksPerPage) brow[pad] = -INFINITY;
        }
      }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// ---------------------------------------------------------------------------
// top-k
// ---------------------------------------------------------------------------

constexpr int kTopkThreads = 1024;
constexpr int kTopkSmemKeys = 16384;   // keys cached in shared memory up to this count
constexpr int kCandCap = 4096;         // boundary-bucket candidates kept for refinement
constexpr int kRankCand = 1024;        // up to this many are ranked by pairwise counting

// Exclusive scan of one value per thread across the CTA (kTopkThreads threads).
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
    uint32_t s = lane < kTopkThreads / 32 ? warp_sums[lane] : 0u;
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

struct __align__(16) TopkSmem {
  uint32_t hist[4096];
  uint32_t cand[kCandCap];
  uint32_t warp_sums[33];
  uint32_t bucket, above, nvalid, ncand;
};

// Histogram increment (plain shared-memory atomics measured faster here than
// aggregating equal bins across a warp with match_any).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool pred) {
  if (pred) atomicAdd(&hist[bin], 1u);
}

// Find the bucket holding the k_rem-th largest element of a histogram of
// `nbins` bins (larger bin = larger key).  Sets sm->bucket and sm->above
// (elements in higher bins).
__device__ __forceinline__ void find_bucket(TopkSmem* sm, int nbins, uint32_t k_rem) {
  const int per = (nbins + kTopkThreads - 1) / kTopkThreads;   // bins per thread
  const int t = threadIdx.x;
  uint32_t local = 0;
  const int hi = nbins - per * t;   // this thread's bins: [hi-per, hi), counted from the top
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
  if (SRC == SRC_CAND) return pool_row[i];
  return (int32_t)i;
}

constexpr int kKeysPerThread = kTopkSmemKeys / kTopkThreads;   // 16
static_assert(kKeysPerThread == 16, "a thread's positions span exactly two 8-token pool blocks");

// Top-k of up to 16,384 entries with every key held in registers: thread t
// owns positions [16t, 16t+16).
//  1. a CTA reduction gives the number of valid keys and their largest and
//     smallest key; all valid keys share the bits above the highest bit where
//     those two differ, so the radix passes start below that common prefix
//     (scores of similar size then spread over the bins instead of piling
//     into a few);
//  2. pass 1 histograms the next up-to-12 bits of every key (shared-memory
//     atomics) and a CTA scan over the bins finds the bucket holding the k-th
//     key; the bucket's keys are gathered into a candidate list (atomic
//     append) and each candidate counts the candidates above and equal to it
//     (or, for a bucket of more than 1,024, further CTA histogram passes
//     refine it), giving the exact k-th largest key T and the number of keys
//     equal to T to keep (the lowest-position ones);
//  3. one CTA scan of per-thread (count > T, count == T) gives every thread
//     its output offset; selected positions are written in position order.
// If the boundary bucket holds more keys than the candidate list, the further
// passes run over all keys (prefix-filtered).
template <int SRC>
__device__ __forceinline__ void topk_registers(const float* __restrict__ srow, int64_t n, int k,
                                               const int32_t* pool_row, int32_t* __restrict__ orow,
                                               float* __restrict__ oscore, int32_t id_off, TopkSmem* sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t lo = (int64_t)tid * kKeysPerThread;
  uint32_t key[kKeysPerThread];
#pragma unroll
  for (int j = 0; j < kKeysPerThread; j += 4) {
    if (lo + j < n) {   // n is a multiple of 8, so a float4 never straddles the end
      const float4 f = *reinterpret_cast<const float4*>(srow + lo + j);
      key[j] = score_key(f.x); key[j + 1] = score_key(f.y);
      key[j + 2] = score_key(f.z); key[j + 3] = score_key(f.w);
    } else {
      key[j] = key[j + 1] = key[j + 2] = key[j + 3] = 0u;
    }
  }
  // pool blocks of this thread's positions (16 positions = 2 blocks), fetched early
  int32_t pb0 = 0, pb1 = 0;
  if (SRC == SRC_POOL && lo < n) {
    pb0 = pool_row[lo >> 3];
    pb1 = pool_row[(lo >> 3) + 1];
  }
  // valid count, largest and smallest valid key
  uint32_t nv = 0, kmax = 0u, kmin = 0xFFFFFFFFu;
#pragma unroll
  for (int j = 0; j < kKeysPerThread; ++j) {
    if (key[j]) {
      ++nv;
      kmax = max(kmax, key[j]);
      kmin = min(kmin, key[j]);
    }
  }
  nv = __reduce_add_sync(0xffffffffu, nv);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  uint32_t* red = sm->cand;   // scratch: [0,32) counts, [32,64) maxima, [64,96) minima
  if (lane == 0) {
    red[warp] = nv;
    red[32 + warp] = kmax;
    red[64 + warp] = kmin;
  }
  for (int i = tid; i < 4096; i += kTopkThreads) sm->hist[i] = 0;
  __syncthreads();
  {
    const bool in = lane < kTopkThreads / 32;
    const uint32_t a = in ? red[lane] : 0u, bmax = in ? red[32 + lane] : 0u,
                   bmin = in ? red[64 + lane] : 0xFFFFFFFFu;
    nv = __reduce_add_sync(0xffffffffu, a);
    kmax = __reduce_max_sync(0xffffffffu, bmax);
    kmin = __reduce_min_sync(0xffffffffu, bmin);
  }
  const uint32_t nvalid = nv;

  uint32_t T = 1u, need_eq = 0xFFFFFFFFu;
  if (nvalid > (uint32_t)k) {
    uint32_t k_rem = (uint32_t)k;
    // bits [0, top) are still open; the bits above are the valid keys' common prefix
    int top = 32 - __clz((int)(kmax ^ kmin));
    uint32_t prefix = kmax & ~((top >= 32) ? 0xFFFFFFFFu : ((1u << top) - 1u));
    if (top == 0) {   // every valid key is equal
      T = kmax;
      need_eq = k_rem;
    } else {
      int width = top < 12 ? top : 12;
      int shift = top - width;
      // pass 1 over every valid key
#pragma unroll
      for (int j = 0; j < kKeysPerThread; ++j)
        if (key[j]) atomicAdd(&sm->hist[(key[j] >> shift) & ((1u << width) - 1u)], 1u);
      __syncthreads();
      find_bucket(sm, 1 << width, k_rem);
      prefix |= sm->bucket << shift;
      k_rem -= sm->above;
      if (shift > 0) {
        // gather the boundary bucket (order does not matter for the selection)
        const uint32_t pmask = ~((1u << shift) - 1u);
        uint32_t nm = 0;
#pragma unroll
        for (int j = 0; j < kKeysPerThread; ++j) nm += (key[j] && (key[j] & pmask) == prefix) ? 1u : 0u;
        if (tid == 0) sm->ncand = 0;
        __syncthreads();
        uint32_t off = nm ? atomicAdd(&sm->ncand, nm) : 0u;
        if (nm) {
#pragma unroll
          for (int j = 0; j < kKeysPerThread; ++j)
            if (key[j] && (key[j] & pmask) == prefix && off < (uint32_t)kCandCap) sm->cand[off++] = key[j];
        }
        __syncthreads();
        const uint32_t ncand = sm->ncand;
        if (ncand <= (uint32_t)kRankCand) {
          // every candidate counts the candidates above and equal to it; the one
          // whose rank brackets k_rem is the k-th largest key T
          if (tid < (int)ncand) {
            const uint32_t c = sm->cand[tid];
            uint32_t gt = 0, eq = 0;
            const uint4* c4 = reinterpret_cast<const uint4*>(sm->cand);
            const uint32_t n4 = ncand >> 2;
            for (uint32_t i = 0; i < n4; ++i) {
              const uint4 x = c4[i];
              gt += (x.x > c) + (x.y > c) + (x.z > c) + (x.w > c);
              eq += (x.x == c) + (x.y == c) + (x.z == c) + (x.w == c);
            }
            for (uint32_t i = n4 << 2; i < ncand; ++i) {
              const uint32_t x = sm->cand[i];
              gt += x > c;
              eq += x == c;
            }
            if (gt < k_rem && gt + eq >= k_rem) {   // equal candidates write the same values
              sm->bucket = c;
              sm->above = k_rem - gt;
            }
          }
          __syncthreads();
          prefix = sm->bucket;
          k_rem = sm->above;
        } else {
          const bool use_cand = ncand <= (uint32_t)kCandCap;
#pragma unroll 1
          while (shift > 0) {
            const uint32_t pm = ~((1u << shift) - 1u);
            width = shift < 12 ? shift : 12;
            shift -= width;
            const uint32_t dmask = (1u << width) - 1u;
            for (int i = tid; i < (1 << width); i += kTopkThreads) sm->hist[i] = 0;
            __syncthreads();
            if (use_cand) {
              for (uint32_t i = tid; i < ncand; i += kTopkThreads) {
                const uint32_t kk = sm->cand[i];
                if ((kk & pm) == prefix) atomicAdd(&sm->hist[(kk >> shift) & dmask], 1u);
              }
            } else {
#pragma unroll
              for (int j = 0; j < kKeysPerThread; ++j)
                if (key[j] && (key[j] & pm) == prefix) atomicAdd(&sm->hist[(key[j] >> shift) & dmask], 1u);
            }
            __syncthreads();
            find_bucket(sm, 1 << width, k_rem);
            prefix |= sm->bucket << shift;
            k_rem -= sm->above;
          }
        }
      }
      T = prefix;
      need_eq = k_rem;
    }
  }
  // output: one scan of packed (count > T, count == T); both fit 16 bits
  uint32_t ngt = 0, neq = 0;
#pragma unroll
  for (int j = 0; j < kKeysPerThread; ++j) {
    ngt += (key[j] != 0u && key[j] > T) ? 1u : 0u;
    neq += (key[j] != 0u && key[j] == T) ? 1u : 0u;
  }
  uint32_t tot;
  const uint32_t before = cta_exclusive_scan((ngt << 16) | neq, sm->warp_sums, &tot);
  const uint32_t gt_before = before >> 16, eq_before = before & 0xFFFFu;
  const uint32_t tot_gt = tot >> 16, tot_eq = tot & 0xFFFFu;
  uint32_t slot = gt_before + min(eq_before, need_eq);
  uint32_t eq_rank = eq_before;
  if (ngt + neq > 0) {   // most threads select nothing
#pragma unroll
    for (int j = 0; j < kKeysPerThread; ++j) {
      const uint32_t kj = key[j];
      bool sel = kj != 0u && kj > T;
      if (kj != 0u && kj == T) sel = eq_rank++ < need_eq;
      if (sel && slot < (uint32_t)k) {
        int32_t o;
        if (SRC == SRC_POOL) o = (j < 8 ? pb0 : pb1) * kBlock + (int32_t)((lo + j) & 7);
        else if (SRC == SRC_CAND) o = pool_row[lo + j];
        else o = (int32_t)(lo + j);
        if (oscore) oscore[slot] = key_score(kj);
        orow[slot++] = o + id_off;
      }
    }
  }
  const uint32_t total = tot_gt + min(tot_eq, need_eq);
  for (int64_t s = (int64_t)total + tid; s < k; s += kTopkThreads) {
    orow[s] = -1;
    if (oscore) oscore[s] = -INFINITY;
  }
}

// One CTA per query: select the k best entries of scores[r][0 .. n_r).
// Up to 16,384 entries: keys in registers (topk_registers).  Larger rows
// (the block level of a 1M context, a long encoder prefix):
//  1. histogram of the keys' top 12 bits (order-preserving uint32 of the
//     scores, 0 = no candidate), read from the workspace;
//  2. the bucket holding the k-th key is found; its keys are compacted into a
//     candidate list and refined on bits 19..8 and 7..0, giving the exact
//     k-th key T and how many keys equal to T are kept;
//  3. each thread takes a contiguous segment of positions, counts its keys
//     above T and equal to T, one CTA scan gives its output offset, and it
//     writes its selected positions in order (ascending overall).
// kRegOnly: the launch guarantees n <= 16,384 for every row, so only the
// register path is compiled (far less code for each launch to fetch).
template <int SRC, bool kRegOnly>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(CacheView c, const float* __restrict__ scores,
                                                            int64_t stride, const int32_t* __restrict__ q_seq,
                                                            const int32_t* __restrict__ q_vis,
                                                            const int32_t* __restrict__ pool, int k,
                                                            TopkOut out) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem* sm = reinterpret_cast<TopkSmem*>(smem_raw);

  const int r = out.nseg > 1 ? (int)(blockIdx.x / out.nseg) : (int)blockIdx.x;
  const int64_t seg0 = out.nseg > 1 ? (int64_t)(blockIdx.x % out.nseg) * out.seg_len : 0;
  const int tid = threadIdx.x;
  // candidates: every entry of the row (a multiple of 8), ids from `pool`; a
  // segment: entries [seg0, seg0 + seg_len) of it
  int64_t n = SRC == SRC_CAND ? stride
                              : min(units_of(SRC, visible_of(c, q_seq, q_vis, r)) * kBlock, stride);
  if (out.nseg > 1) n = n - seg0 < 0 ? 0 : (n - seg0 < out.seg_len ? n - seg0 : out.seg_len);
  const float* srow = scores + (int64_t)r * stride + seg0;
  const int32_t* pool_row =
      pool ? pool + (int64_t)r * (SRC == SRC_CAND ? stride : (int64_t)kPoolBlocks) : nullptr;
  int32_t* orow = out.ids + (int64_t)blockIdx.x * out.stride;
  float* oscore = out.scores ? out.scores + (int64_t)blockIdx.x * out.stride : nullptr;
  const int32_t id_off = (out.id_offset ? (out.id_offset[r] >> out.offset_shift) : 0) + (int32_t)seg0;
  if (kRegOnly || n <= kTopkSmemKeys) {
    topk_registers<SRC>(srow, n, k, pool_row, orow, oscore, id_off, sm);
    return;
  }
  auto key_at = [&](int64_t i) -> uint32_t { return score_key(srow[i]); };

  // pass 0: valid count, histogram of bits 31..20
  for (int i = tid; i < 4096; i += kTopkThreads) sm->hist[i] = 0;
  if (tid == 0) {
    sm->nvalid = 0;
    sm->ncand = 0;
  }
  __syncthreads();
  uint32_t myvalid = 0;
  for (int64_t b0 = 0; b0 < n; b0 += 4 * kTopkThreads) {
    const int64_t i4 = b0 + 4 * (int64_t)tid;
    uint32_t kk[4] = {0u, 0u, 0u, 0u};
    if (i4 < n) {
      const float4 f = *reinterpret_cast<const float4*>(srow + i4);
      kk[0] = score_key(f.x); kk[1] = score_key(f.y); kk[2] = score_key(f.z); kk[3] = score_key(f.w);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      myvalid += kk[j] ? 1u : 0u;
      hist_add(sm->hist, kk[j] >> 20, kk[j] != 0u);
    }
  }
  atomicAdd(&sm->nvalid, myvalid);
  __syncthreads();
  const uint32_t nvalid = sm->nvalid;

  uint32_t T = 1u;                  // keep every key > T ...
  uint32_t need_eq = 0xFFFFFFFFu;   // ... and this many keys == T (lowest positions first)
  if (nvalid > (uint32_t)k) {
    uint32_t k_rem = (uint32_t)k;
    find_bucket(sm, 4096, k_rem);
    const uint32_t b1 = sm->bucket;
    k_rem -= sm->above;
    // compact the boundary bucket's keys
    for (int64_t b0 = 0; b0 < n; b0 += kTopkThreads) {
      const int64_t i = b0 + tid;
      const uint32_t key = i < n ? key_at(i) : 0u;
      const bool m = key != 0u && (key >> 20) == b1;
      const uint32_t bal = __ballot_sync(0xffffffffu, m);
      uint32_t base = 0;
      if ((tid & 31) == 0 && bal) base = atomicAdd(&sm->ncand, (uint32_t)__popc(bal));
      base = __shfl_sync(0xffffffffu, base, 0);
      const uint32_t slot = base + __popc(bal & ((1u << (tid & 31)) - 1u));
      if (m && slot < (uint32_t)kCandCap) sm->cand[slot] = key;
    }
    __syncthreads();
    const uint32_t ncand = sm->ncand;
    const bool use_cand = ncand <= (uint32_t)kCandCap;
    // refine on bits 19..8, then 7..0 (over the candidates, or over all keys
    // with the bucket prefix when the bucket overflowed the candidate list)
    uint32_t prefix = b1 << 20;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 8 : 0;
      const uint32_t pmask = pass == 0 ? 0xFFF00000u : 0xFFFFFF00u;
      const uint32_t dmask = pass == 0 ? 0xFFFu : 0xFFu;
      for (int i = tid; i < 4096; i += kTopkThreads) sm->hist[i] = 0;
      __syncthreads();
      const int64_t m_n = use_cand ? (int64_t)ncand : n;
      for (int64_t b0 = 0; b0 < m_n; b0 += kTopkThreads) {
        const int64_t i = b0 + tid;
        const uint32_t key = i < m_n ? (use_cand ? sm->cand[i] : key_at(i)) : 0u;
        hist_add(sm->hist, (key >> shift) & dmask, key != 0u && (key & pmask) == prefix);
      }
      __syncthreads();
      find_bucket(sm, pass == 0 ? 4096 : 256, k_rem);
      prefix |= sm->bucket << shift;
      k_rem -= sm->above;
    }
    T = prefix;
    need_eq = k_rem;
  }

  // output: contiguous segments in position order (read 4 keys at a time)
  const int64_t seg = (((n + kTopkThreads - 1) / kTopkThreads) + 3) & ~(int64_t)3;
  const int64_t lo = min((int64_t)tid * seg, n), hi = min(lo + seg, n);
  uint32_t ngt = 0, neq = 0;
  for (int64_t i = lo; i < hi; i += 4) {
    const float4 f = *reinterpret_cast<const float4*>(srow + i);
    const uint32_t kk[4] = {score_key(f.x), score_key(f.y), score_key(f.z), score_key(f.w)};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      ngt += (kk[j] != 0u && kk[j] > T) ? 1u : 0u;
      neq += (kk[j] != 0u && kk[j] == T) ? 1u : 0u;
    }
  }
  uint32_t tot_gt, tot_eq;
  const uint32_t gt_before = cta_exclusive_scan(ngt, sm->warp_sums, &tot_gt);
  const uint32_t eq_before = cta_exclusive_scan(neq, sm->warp_sums, &tot_eq);
  uint32_t slot = gt_before + min(eq_before, need_eq);
  uint32_t eq_rank = eq_before;
  if (ngt + neq > 0) {
    for (int64_t i = lo; i < hi; i += 4) {
      const float4 f = *reinterpret_cast<const float4*>(srow + i);
      const uint32_t kk[4] = {score_key(f.x), score_key(f.y), score_key(f.z), score_key(f.w)};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (kk[j] == 0u || kk[j] < T) continue;
        bool sel = kk[j] > T;
        if (!sel) sel = eq_rank++ < need_eq;
        if (sel && slot < (uint32_t)k) {
          if (oscore) oscore[slot] = key_score(kk[j]);
          orow[slot++] = map_out<SRC>(i + j, pool_row) + id_off;
        }
      }
    }
  }
  const uint32_t total = tot_gt + min(tot_eq, need_eq);
  for (int64_t s = (int64_t)total + tid; s < k; s += kTopkThreads) {
    orow[s] = -1;
    if (oscore) oscore[s] = -INFINITY;
  }
}

}  // namespace csa2

// ---- launchers used by api.cu ----
namespace csa2 {

size_t topk_smem_bytes() { return sizeof(TopkSmem); }

cudaError_t score_mma_set_attributes();
cudaError_t launch_score_mma(int src, const CacheView& c, const uint16_t* idx_q, const float* head_w,
                             const int32_t* q_seq, const int32_t* q_vis, const int32_t* pool, int nq,
                             int64_t max_units, int64_t stride, float* scores, float* block_max, int64_t bstride,
                             cudaStream_t st);

// Opt the top-k kernels in to their shared-memory size (once per device).
cudaError_t indexer_set_attributes() {
  const int smem = (int)topk_smem_bytes();
  const void* topk_kernels[] = {
      (const void*)topk_kernel<SRC_FLAT, false>,      (const void*)topk_kernel<SRC_FLAT, true>,
      (const void*)topk_kernel<SRC_BLOCKKEYS, false>, (const void*)topk_kernel<SRC_BLOCKKEYS, true>,
      (const void*)topk_kernel<SRC_POOL, true>,       (const void*)topk_kernel<SRC_CAND, false>,
      (const void*)topk_kernel<SRC_CAND, true>};
  cudaError_t e = cudaSuccess;
  for (const void* k : topk_kernels)
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const void* score_kernels[] = {(const void*)score_units_kernel<SRC_FLAT, true>,
                                 (const void*)score_units_kernel<SRC_POOL, true>};
  for (const void* k : score_kernels)
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScoreSmemMax);
  if (e == cudaSuccess) e = score_mma_set_attributes();
  return e;
}

// Scores of every query's units into `scores` (row stride `stride` floats).
cudaError_t launch_score(int src, const CacheView& c, const uint16_t* idx_q, const float* head_w,
                         const int32_t* q_seq, const int32_t* q_vis, const int32_t* pool, int nq,
                         int64_t max_units, int64_t stride, float* scores, float* block_max,
                         int64_t bstride, cudaStream_t st) {
  // bf16 keys (and block keys, always bf16): tensor-core scoring (score_mma.cu);
  // FP8 keys: the FFMA kernel below
  if (!c.idxk_fp8 || src == SRC_BLOCKKEYS)
    return launch_score_mma(src, c, idx_q, head_w, q_seq, q_vis, pool, nq, max_units, stride, scores, block_max,
                            bstride, st);
  // units per CTA: enough CTAs for two per SM over the whole batch, in whole
  // 32-unit stages, at most 256
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t per_query = nq > 0 ? ((int64_t)2 * sms) / nq : 1;   // CTAs per query that fit in one wave
  if (per_query < 1) per_query = 1;
  int64_t upc = (max_units + per_query - 1) / per_query;
  const int stage_units = ScoreGeom<true>::kUnits;
  const uint32_t smem = ScoreGeom<true>::kSmem;
  upc = (upc + stage_units - 1) / stage_units * stage_units;
  if (upc > kUnitsPerCta) upc = kUnitsPerCta;
  if (upc < stage_units) upc = stage_units;
  dim3 grid((unsigned)((max_units + upc - 1) / upc), (unsigned)nq);
  if (grid.x == 0) return cudaSuccess;
  if (src == SRC_FLAT)
    launch_pdl(score_units_kernel<SRC_FLAT, true>, grid, kScoreThreads, smem, st, c, idx_q, head_w, q_seq, q_vis,
               pool, max_units, stride, (int)upc, scores, block_max, bstride);
  else
    launch_pdl(score_units_kernel<SRC_POOL, true>, grid, kScoreThreads, smem, st, c, idx_q, head_w, q_seq, q_vis,
               pool, max_units, stride, (int)upc, scores, block_max, bstride);
  return cudaGetLastError();
}

cudaError_t launch_topk(int src, const CacheView& c, const float* scores, int64_t stride,
                        const int32_t* q_seq, const int32_t* q_vis, const int32_t* pool, int nq,
                        int k, int32_t* out, int64_t out_stride, cudaStream_t st, float* out_scores,
                        const int32_t* id_offset, int offset_shift, int nseg) {
  const size_t smem = topk_smem_bytes();
  if (nq == 0) return cudaSuccess;
  // nseg > 1: one CTA per segment of kTopkSmemKeys entries; output rows nq x nseg
  const TopkOut o{out, out_stride, out_scores, id_offset, offset_shift, nseg > 1 ? nseg : 1, kTopkSmemKeys};
  if (nseg > 1) nq *= nseg;
  // every row fits the register path when a row holds at most 16,384 entries:
  // n <= stride always, n <= the segment length when segmented, and a pool row
  // is 2,048 blocks x 8 tokens
  const bool reg = nseg > 1 || src == SRC_POOL || stride <= kTopkSmemKeys;
#define CSA2_TOPK_LAUNCH(S, R) \
  launch_pdl(topk_kernel<S, R>, nq, kTopkThreads, smem, st, c, scores, stride, q_seq, q_vis, pool, k, o)
  if (src == SRC_FLAT) {
    if (reg) CSA2_TOPK_LAUNCH(SRC_FLAT, true);
    else CSA2_TOPK_LAUNCH(SRC_FLAT, false);
  } else if (src == SRC_BLOCKKEYS) {
    if (reg) CSA2_TOPK_LAUNCH(SRC_BLOCKKEYS, true);
    else CSA2_TOPK_LAUNCH(SRC_BLOCKKEYS, false);
  } else if (src == SRC_POOL) {
    CSA2_TOPK_LAUNCH(SRC_POOL, true);
  } else {
    if (reg) CSA2_TOPK_LAUNCH(SRC_CAND, true);
    else CSA2_TOPK_LAUNCH(SRC_CAND, false);
  }
#undef CSA2_TOPK_LAUNCH
  return cudaGetLastError();
}

}  // namespace csa2
