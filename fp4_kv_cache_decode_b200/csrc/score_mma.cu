// Indexer scoring on the 5th-generation tensor cores (bf16 indexer keys).
//
// score(q, k) = sum_h w_h * max(0, q_h . k) over 4 heads of 64 dims
// (agentnet.co.il, "דיפסיק משיקה את V4.1-פלאש ...", section "CSA2: דחיסה
// לאורך ציר השכבות": the Full layer's indexer, the block level of the
// hierarchy, and the Reindex layer's ranking of the pool).  The key set of a
// query is a list of 1-KiB units of eight 128-B keys that are contiguous in
// HBM (8 tokens of an indexer-key page, the 8 block keys of a page, or the 8
// tokens of a pool block).  Per CTA (one query, up to 256 units):
//   * the producer warp loads each unit with one TMA tile copy (box 8 keys x
//     64 dims; lane j issues unit j of a tile) straight into the
//     128-byte-swizzled K-major layout the tensor core reads; 16 units make a
//     128-key tile, and 4 tiles are in flight;
//   * one MMA thread issues D[128 keys x 16] = K[128 x 64] . Q^T[64 x 16]
//     (tcgen05.mma kind::f16, bf16 operands, fp32 accumulation in TMEM; Q^T
//     holds the 4 heads in columns 0..3, zeros in 4..15) as 4 K-steps of 16;
//   * four epilogue warps read their 32 keys' 4 head dots with one tcgen05.ld,
//     finish the score in registers and store it (128 consecutive floats per
//     tile), plus, for the flat source, each block's maximum.
// The products are exact (bf16 x bf16) and the sums fp32, so the scores agree
// with the FFMA form up to the order of the fp32 additions.
// Hand-offs use mbarriers: full (TMA bytes), done (tcgen05.commit), free (the
// epilogue has read the accumulator, so the stage's shared memory and TMEM
// columns may be reused).  Every wait is bounded and reports
// CSA2_DEVERR_TIMEOUT; the producer and the MMA thread drain what they issued
// before the CTA frees its tensor memory.
#include <cuda.h>

#include "common.cuh"
#include "indexer.cuh"
#include "tc.cuh"

namespace csa2 {

constexpr int kSmThreads = 192;              // warps 0..3 epilogue, 4 producer, 5 MMA
constexpr int kTileUnits = 16;               // 16 units x 8 keys = 128 keys = MMA M
constexpr int kSmStages = 4;
constexpr int kSmUnitsPerCta = 256;
constexpr uint32_t kTileBytesS = kTileUnits * 1024u;
constexpr uint32_t kSmTmemCols = 64;         // kSmStages accumulators of 16 columns
constexpr uint32_t kSmOffA = 0;                                    // [stages][16 KiB]
constexpr uint32_t kSmOffB = kSmStages * kTileBytesS;              // Q^T [16 x 64] bf16, 2 KiB
constexpr uint32_t kSmOffRow = kSmOffB + 2048;                     // int32 TMA row per unit (-1: none)
constexpr uint32_t kSmOffNr = kSmOffRow + 4 * kSmUnitsPerCta;      // int32 valid keys per unit
constexpr uint32_t kSmOffBar = kSmOffNr + 4 * kSmUnitsPerCta;      // full / done / free per stage
constexpr uint32_t kSmOffMisc = kSmOffBar + 8 * 3 * kSmStages;     // TMEM base, abort flag
constexpr uint32_t kScoreMmaSmem = kSmOffMisc + 16 + 1024;         // + slack for 1024-B alignment
// tcgen05.mma kind::f16 instruction descriptor: D fp32 (bit 4), A and B bf16
// (bits 7, 10), both K-major, N = 16 (N >> 3 at bit 17), M = 128 (M >> 4 at bit 24)
constexpr uint32_t kIdescScore = (1u << 4) | (1u << 7) | (1u << 10) | ((16u >> 3) << 17) | ((128u >> 4) << 24);
static_assert(kScoreMmaSmem <= 232448 / 3, "three CTAs per SM");

template <int SRC>
__global__ void __launch_bounds__(kSmThreads) score_mma_kernel(const __grid_constant__ CUtensorMap tmap, CacheView c,
                                                               const uint16_t* __restrict__ idx_q,
                                                               const float* __restrict__ head_w,
                                                               const int32_t* __restrict__ q_seq,
                                                               const int32_t* __restrict__ q_vis,
                                                               const int32_t* __restrict__ pool, int64_t max_units,
                                                               int64_t stride, int upc, float* __restrict__ scores,
                                                               float* __restrict__ block_max, int64_t bstride) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw = (uint32_t)__cvta_generic_to_shared(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;   // 1024-B aligned: the swizzle atoms of A and B
  uint8_t* const sp = smem_raw + (sb - raw);
  const int r = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int seq = q_seq[r];
  const int64_t v = visible_of(c, q_seq, q_vis, r);
  int64_t nunits = units_of(SRC, v);
  if (nunits > max_units) {
    if (blockIdx.x == 0 && tid == 0) raise_error(c.err, CSA2_DEVERR_POS);
    nunits = max_units;
  }
  const int64_t u0 = (int64_t)blockIdx.x * upc;
  if (u0 >= nunits) return;
  const int nu = (int)(nunits - u0 < upc ? nunits - u0 : upc);
  const int ntiles = (nu + kTileUnits - 1) / kTileUnits;
  const int64_t nb = (v + kBlock - 1) / kBlock;
  int32_t* const urow = reinterpret_cast<int32_t*>(sp + kSmOffRow);
  int32_t* const unr = reinterpret_cast<int32_t*>(sp + kSmOffNr);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(sp + kSmOffMisc + 4);
  auto full = [&](int s) { return sb + kSmOffBar + 8u * s; };
  auto done = [&](int s) { return sb + kSmOffBar + 8u * (kSmStages + s); };
  auto freed = [&](int s) { return sb + kSmOffBar + 8u * (2 * kSmStages + s); };

  // unit rows of the tensor map (keys: page x 64 + slot; block keys: page x 8)
  for (int j = tid; j < kSmUnitsPerCta; j += kSmThreads) {
    int32_t row = -1, nr = 0;
    if (j < nu) {
      const int64_t u = u0 + j;
      if (SRC == SRC_FLAT) {
        const int64_t pg = page_of(c, seq, u * kBlock);
        if (pg >= 0) {
          row = (int32_t)(pg * kPageTokens + (u & (kBlocksPerPage - 1)) * kBlock);
          nr = (int)(v - u * kBlock < kBlock ? v - u * kBlock : kBlock);
        }
      } else if (SRC == SRC_BLOCKKEYS) {
        const int64_t pg = page_of(c, seq, u * kPageTokens);
        if (pg >= 0) {
          row = (int32_t)(pg * kBlocksPerPage);
          nr = (int)(nb - u * kBlocksPerPage < kBlocksPerPage ? nb - u * kBlocksPerPage : kBlocksPerPage);
        }
      } else {
        const int32_t blk = pool[(int64_t)r * kPoolBlocks + u];
        if (blk >= 0) {
          if ((int64_t)blk >= nb) {
            raise_error(c.err, CSA2_DEVERR_POS);
          } else {
            const int64_t pg = page_of(c, seq, (int64_t)blk * kBlock);
            if (pg >= 0) {
              row = (int32_t)(pg * kPageTokens + (blk & (kBlocksPerPage - 1)) * kBlock);
              nr = (int)(v - (int64_t)blk * kBlock < kBlock ? v - (int64_t)blk * kBlock : kBlock);
            }
          }
        }
      }
    }
    urow[j] = row;
    unr[j] = nr;
  }
  // Q^T: row h = head h (rows 4..15 zero), 128-B swizzled K-major
  for (int i = tid; i < 16 * 8; i += kSmThreads) {
    const int h = i >> 3, ch = i & 7;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (h < kIdxHeads) val = __ldg(reinterpret_cast<const uint4*>(idx_q + ((int64_t)r * kIdxHeads + h) * kIdxDim) + ch);
    *reinterpret_cast<uint4*>(sp + kSmOffB + h * 128 + ((ch ^ (h & 7)) << 4)) = val;
  }
  fence_async_smem();   // the tensor core reads Q^T through the async proxy
  if (tid == 0) {
    for (int s = 0; s < kSmStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(done(s), 1);
      mbar_init(freed(s), 4);
    }
    *abort_flag = 0;
#ifdef CSA2_TEST_HOOKS
    mbar_init(sb + kSmOffMisc + 8, 1);   // completed by nothing: the test stall waits on it
#endif
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) tmem_alloc_warp(sb + kSmOffMisc, kSmTmemCols);
  if (warp == 4 && lane == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap)) : "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sp + kSmOffMisc);

  if (warp == 4) {
    // ---- producer warp: lane j issues the TMA copy of unit j of each tile (one
    // issuing thread per unit: a single thread spends ~0.1 us per tensor copy) ----
    int t = 0;
#pragma unroll 1
    for (; t < ntiles; ++t) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const int s = t % kSmStages, n = t / kSmStages;
      bool ok = true;
      if (n > 0) ok = __all_sync(0xffffffffu, lane != 0 || mbar_wait(freed(s), (n - 1) & 1));
      if (!ok) {
        if (lane == 0) {
          *abort_flag = 1;
          raise_error(c.err, CSA2_DEVERR_TIMEOUT);
        }
        break;
      }
      // flat: a tile's 16 units are two whole pages (u0 and the tiles start at
      // multiples of 16 units), one 64-key box each; otherwise one 8-key box per unit
      constexpr int kBoxUnits = SRC == SRC_FLAT ? kBlocksPerPage : 1;
      const int uj = t * kTileUnits + lane * kBoxUnits;
      const int32_t row = (lane < kTileUnits / kBoxUnits && uj < nu) ? urow[uj] : -1;
      const uint32_t mask = __ballot_sync(0xffffffffu, row >= 0);
      if (lane == 0) mbar_arrive_expect_tx(full(s), (uint32_t)__popc(mask) * 1024u * kBoxUnits);
      __syncwarp();
      if (row >= 0)
        tma_load_2d(sb + kSmOffA + (uint32_t)s * kTileBytesS + (uint32_t)(lane * kBoxUnits) * 1024u, &tmap, 0, row,
                    full(s));
      __syncwarp();
    }
    // every stage's last copy lands before the CTA may exit
    if (lane == 0)
      for (int k = (t > kSmStages ? t - kSmStages : 0); k < t; ++k)
        mbar_wait(full(k % kSmStages), (k / kSmStages) & 1);
  } else if (warp == 5) {
    // ---- MMA issue ----
    if (lane == 0) {
      const uint64_t bdesc = smem_desc(sb + kSmOffB, 16, 1024);
      int t = 0;
#ifdef CSA2_TEST_HOOKS
      // test stall before the first MMA: the wait runs out, the CTA aborts
      if (test_stall(c.err) && !test_stall_wait(sb + kSmOffMisc + 8)) {
        *abort_flag = 1;
        raise_error(c.err, CSA2_DEVERR_TIMEOUT);
      }
#endif
      for (; t < ntiles; ++t) {
        if (*abort_flag) break;
        const int s = t % kSmStages, n = t / kSmStages;
        bool ok = mbar_wait(full(s), n & 1);
        if (ok && n > 0) ok = mbar_wait(freed(s), (n - 1) & 1);   // accumulator s read out
        if (!ok) {
          *abort_flag = 1;
          raise_error(c.err, CSA2_DEVERR_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint64_t adesc = smem_desc(sb + kSmOffA + (uint32_t)s * kTileBytesS, 16, 1024);
#pragma unroll
        for (int k = 0; k < kIdxDim / 16; ++k)   // K-steps of 16 bf16 = 32 B along the swizzled row
          mma_f16(tmem + (uint32_t)s * 16u, adesc + 2u * k, bdesc + 2u * k, kIdescScore, k > 0 ? 1u : 0u);
        mma_commit(done(s));
      }
      if (t > 0) mbar_wait(done((t - 1) % kSmStages), ((t - 1) / kSmStages) & 1);   // last MMAs finished
    }
  } else {
    // ---- epilogue: warps 0..3 own TMEM lanes 32 warp .. 32 warp + 31 ----
    float wv[kIdxHeads];
#pragma unroll
    for (int h = 0; h < kIdxHeads; ++h) wv[h] = head_w ? __ldg(head_w + (int64_t)r * kIdxHeads + h) : 1.0f;
    const int row = 32 * warp + lane;   // key within the tile
    float* const srow = scores + (int64_t)r * stride;
    float* const brow = block_max ? block_max + (int64_t)r * bstride : nullptr;
    for (int t = 0; t < ntiles; ++t) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;   // warp-uniform: the loads below are .aligned
      const int s = t % kSmStages, n = t / kSmStages;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(done(s), n & 1));
      if (!ok) {
        if (lane == 0) {
          *abort_flag = 1;
          raise_error(c.err, CSA2_DEVERR_TIMEOUT);
        }
        break;
      }
      tc_fence_after();
      const float4 d = tmem_ld4(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)s * 16u);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(freed(s));
      const int j = t * kTileUnits + (row >> 3);   // unit within the CTA
      const int64_t u = u0 + j;
      float sc = __fmul_rn(wv[0], fmaxf(d.x, 0.0f));
      sc = __fadd_rn(sc, __fmul_rn(wv[1], fmaxf(d.y, 0.0f)));
      sc = __fadd_rn(sc, __fmul_rn(wv[2], fmaxf(d.z, 0.0f)));
      sc = __fadd_rn(sc, __fmul_rn(wv[3], fmaxf(d.w, 0.0f)));
      const bool in = j < nu;
      const float val = (in && (row & 7) < unr[in ? j : 0]) ? sc : -INFINITY;
      if (in) srow[u * kBlock + (row & 7)] = val;
      if (SRC == SRC_FLAT && brow != nullptr) {   // max-pooled block score of block u
        float m = fmaxf(val, __shfl_xor_sync(0xffffffffu, val, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        if (in && (lane & 7) == 0) brow[u] = m;
        // the last block pads the row to a whole unit of 8 block scores with -inf
        if (in && u == nunits - 1 && (lane & 7) == 0) {
          const int64_t end = (nunits + kBlocksPerPage - 1) / kBlocksPerPage * kBlocksPerPage;
          for (int64_t p = nunits; p < end; ++p) brow[p] = -INFINITY;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc_warp(tmem, kSmTmemCols);
  }
}

// ---- flat scoring of query groups ----
//
// Many queries of one sequence (an encoder prefill chunk: consecutive positions,
// visible lengths within a few entries of each other) share their keys: a CTA
// takes 16 consecutive queries, and D[128 keys x 64] = K . Q^T with the 16
// queries' 4 heads as the 64 columns, so each key tile is loaded once for all 16
// and the tensor core does 16x the work per copy.  Each query masks the keys at
// or beyond its own visible length.  A group whose queries are not all of one
// sequence is scored one query per pass (same Q^T, that query's 4 columns).
constexpr int kGrp = 16;                                 // queries per CTA
constexpr int kGrpN = kGrp * kIdxHeads;                  // 64 = MMA N
constexpr uint32_t kGrpTmemCols = kSmStages * kGrpN;     // 256
constexpr uint32_t kGrOffA = 0;                          // [stages][16 KiB]
constexpr uint32_t kGrOffB = kSmStages * kTileBytesS;    // Q^T [64 x 64] bf16, 8 KiB
constexpr uint32_t kGrOffRow = kGrOffB + 8192;
constexpr uint32_t kGrOffNr = kGrOffRow + 4 * kSmUnitsPerCta;
constexpr uint32_t kGrOffQv = kGrOffNr + 4 * kSmUnitsPerCta;   // int64 visible length per query
constexpr uint32_t kGrOffW = kGrOffQv + 8 * kGrp;              // float head weights [16][4]
constexpr uint32_t kGrOffBar = kGrOffW + 4 * kGrpN;
constexpr uint32_t kGrOffMisc = kGrOffBar + 8 * 3 * kSmStages;  // TMEM base, abort flag, one-sequence flag
// two CTAs per SM hold 2 x 256 TMEM columns; the shared-memory request keeps a third off the SM
constexpr uint32_t kGrpSmem = 232448 / 2 - 1024;
static_assert(kGrOffMisc + 16 + 1024 <= kGrpSmem, "group layout");
static_assert(2 * (kGrpSmem + 1024) <= 233472 && 3 * (kGrpSmem + 1024) > 233472, "two CTAs per SM");
constexpr uint32_t kIdescGrp = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kGrpN >> 3) << 17) | ((128u >> 4) << 24);

__global__ void __launch_bounds__(kSmThreads, 1) score_mma_group_kernel(
    const __grid_constant__ CUtensorMap tmap, CacheView c, const uint16_t* __restrict__ idx_q,
    const float* __restrict__ head_w, const int32_t* __restrict__ q_seq, const int32_t* __restrict__ q_vis, int nq,
    int64_t max_units, int64_t stride, int upc, float* __restrict__ scores) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw = (uint32_t)__cvta_generic_to_shared(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* const sp = smem_raw + (sb - raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r0 = blockIdx.y * kGrp;
  const int ng = nq - r0 < kGrp ? nq - r0 : kGrp;
  int32_t* const urow = reinterpret_cast<int32_t*>(sp + kGrOffRow);
  int32_t* const unr = reinterpret_cast<int32_t*>(sp + kGrOffNr);
  int64_t* const qv = reinterpret_cast<int64_t*>(sp + kGrOffQv);
  float* const wq = reinterpret_cast<float*>(sp + kGrOffW);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(sp + kGrOffMisc + 4);
  volatile int* const one_seq = reinterpret_cast<volatile int*>(sp + kGrOffMisc + 8);
  auto full = [&](int s) { return sb + kGrOffBar + 8u * s; };
  auto done = [&](int s) { return sb + kGrOffBar + 8u * (kSmStages + s); };
  auto freed = [&](int s) { return sb + kGrOffBar + 8u * (2 * kSmStages + s); };

  if (tid < kGrp) qv[tid] = tid < ng ? visible_of(c, q_seq, q_vis, r0 + tid) : -1;
  if (tid < kGrpN)
    wq[tid] = (head_w != nullptr && (tid >> 2) < ng) ? __ldg(head_w + (int64_t)(r0 + (tid >> 2)) * kIdxHeads + (tid & 3))
                                                     : 1.0f;
  if (warp == 0) {
    const int32_t s0 = q_seq[r0];
    const bool same = __all_sync(0xffffffffu, lane >= ng || q_seq[r0 + lane] == s0);
    if (lane == 0) *one_seq = same ? 1 : 0;
  }
  // Q^T: row 4 q + h = head h of query q (zero rows past the group), 128-B swizzled K-major
  for (int i = tid; i < kGrpN * 8; i += kSmThreads) {
    const int n = i >> 3, ch = i & 7, q = n >> 2, h = n & 3;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (q < ng) val = __ldg(reinterpret_cast<const uint4*>(idx_q + ((int64_t)(r0 + q) * kIdxHeads + h) * kIdxDim) + ch);
    *reinterpret_cast<uint4*>(sp + kGrOffB + n * 128 + ((ch ^ (n & 7)) << 4)) = val;
  }
  fence_async_smem();
  if (tid == 0) {
    for (int s = 0; s < kSmStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(done(s), 1);
      mbar_init(freed(s), 4);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) tmem_alloc_warp(sb + kGrOffMisc, kGrpTmemCols);
  if (warp == 4 && lane == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap)) : "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sp + kGrOffMisc);
  const bool uniform = *one_seq != 0;
  const int npass = uniform ? 1 : ng;
  const int64_t u0 = (int64_t)blockIdx.x * upc;
  int tbase = 0;          // tiles of earlier passes: the stage / phase count runs on across passes
  int issued = 0, mmas = 0;   // tiles copied / multiplied (for the drains)

#pragma unroll 1
  for (int pass = 0; pass < npass; ++pass) {
    if (*abort_flag) break;   // read after a barrier: the same value in every thread
    const int rq = uniform ? r0 : r0 + pass;
    const int seq = q_seq[rq];
    int64_t v = 0;
    if (uniform) {
      for (int q = 0; q < ng; ++q) v = qv[q] > v ? qv[q] : v;
    } else {
      v = qv[pass];
    }
    int64_t nunits = units_of(SRC_FLAT, v);
    if (nunits > max_units) {
      if (blockIdx.x == 0 && tid == 0) raise_error(c.err, CSA2_DEVERR_POS);
      nunits = max_units;
    }
    const int nu = u0 < nunits ? (int)(nunits - u0 < upc ? nunits - u0 : upc) : 0;
    const int ntiles = (nu + kTileUnits - 1) / kTileUnits;
    for (int j = tid; j < kSmUnitsPerCta; j += kSmThreads) {
      int32_t row = -1, nr = 0;
      if (j < nu) {
        const int64_t u = u0 + j;
        const int64_t pg = page_of(c, seq, u * kBlock);
        if (pg >= 0) {
          row = (int32_t)(pg * kPageTokens + (u & (kBlocksPerPage - 1)) * kBlock);
          nr = (int)(v - u * kBlock < kBlock ? v - u * kBlock : kBlock);
        }
      }
      urow[j] = row;
      unr[j] = nr;
    }
    __syncthreads();

    if (warp == 4) {
      // ---- producer warp: one 64-key box (a whole page) per lane 0 / 1 of each tile ----
      for (int t = 0; t < ntiles; ++t) {
        if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
        const int tg = tbase + t, s = tg % kSmStages, n = tg / kSmStages;
        bool ok = true;
        if (n > 0) ok = __all_sync(0xffffffffu, lane != 0 || mbar_wait(freed(s), (n - 1) & 1));
        if (!ok) {
          if (lane == 0) {
            *abort_flag = 1;
            raise_error(c.err, CSA2_DEVERR_TIMEOUT);
          }
          break;
        }
        const int uj = t * kTileUnits + lane * kBlocksPerPage;
        const int32_t row = (lane < kTileUnits / kBlocksPerPage && uj < nu) ? urow[uj] : -1;
        const uint32_t mask = __ballot_sync(0xffffffffu, row >= 0);
        if (lane == 0) mbar_arrive_expect_tx(full(s), (uint32_t)__popc(mask) * 1024u * kBlocksPerPage);
        __syncwarp();
        if (row >= 0)
          tma_load_2d(sb + kGrOffA + (uint32_t)s * kTileBytesS + (uint32_t)(lane * kBlocksPerPage) * 1024u, &tmap, 0,
                      row, full(s));
        __syncwarp();
        ++issued;
      }
    } else if (warp == 5) {
      // ---- MMA issue ----
      if (lane == 0) {
        const uint64_t bdesc = smem_desc(sb + kGrOffB, 16, 1024);
        for (int t = 0; t < ntiles; ++t) {
          if (*abort_flag) break;
          const int tg = tbase + t, s = tg % kSmStages, n = tg / kSmStages;
          bool ok = mbar_wait(full(s), n & 1);
          if (ok && n > 0) ok = mbar_wait(freed(s), (n - 1) & 1);
          if (!ok) {
            *abort_flag = 1;
            raise_error(c.err, CSA2_DEVERR_TIMEOUT);
            break;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc(sb + kGrOffA + (uint32_t)s * kTileBytesS, 16, 1024);
#pragma unroll
          for (int k = 0; k < kIdxDim / 16; ++k)
            mma_f16(tmem + (uint32_t)s * kGrpN, adesc + 2u * k, bdesc + 2u * k, kIdescGrp, k > 0 ? 1u : 0u);
          mma_commit(done(s));
          ++mmas;
        }
      }
    } else {
      // ---- epilogue: warps 0..3 own TMEM lanes 32 warp .. 32 warp + 31 ----
      const int row = 32 * warp + lane;
      for (int t = 0; t < ntiles; ++t) {
        if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
        const int tg = tbase + t, s = tg % kSmStages, n = tg / kSmStages;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(done(s), n & 1));
        if (!ok) {
          if (lane == 0) {
            *abort_flag = 1;
            raise_error(c.err, CSA2_DEVERR_TIMEOUT);
          }
          break;
        }
        tc_fence_after();
        const int j = t * kTileUnits + (row >> 3);
        const bool in = j < nu;
        const int64_t pos = (u0 + j) * kBlock + (row & 7);
        const bool key_ok = in && (row & 7) < unr[in ? j : 0];
        const uint32_t tbase_addr = tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)s * kGrpN;
        const int q_lo = uniform ? 0 : pass, q_hi = uniform ? ng : pass + 1;
#pragma unroll 1
        for (int q4 = q_lo & ~3; q4 < q_hi; q4 += 4) {   // 4 queries (16 columns) per load
          float d[16];
          tmem_ld16(tbase_addr + 4u * q4, d);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int q = q4 + k;
            if (q < q_lo || q >= q_hi) continue;
            const float* w = wq + 4 * q;
            float sc = __fmul_rn(w[0], fmaxf(d[4 * k], 0.0f));
            sc = __fadd_rn(sc, __fmul_rn(w[1], fmaxf(d[4 * k + 1], 0.0f)));
            sc = __fadd_rn(sc, __fmul_rn(w[2], fmaxf(d[4 * k + 2], 0.0f)));
            sc = __fadd_rn(sc, __fmul_rn(w[3], fmaxf(d[4 * k + 3], 0.0f)));
            if (in) scores[(int64_t)(r0 + q) * stride + pos] = (key_ok && pos < qv[q]) ? sc : -INFINITY;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(freed(s));
      }
    }
    tbase += ntiles;
    __syncthreads();   // the next pass rewrites the unit lists
  }
  // drains: every issued copy has landed and every MMA has finished before the exit
  if (warp == 4 && lane == 0)
    for (int k = (issued > kSmStages ? issued - kSmStages : 0); k < issued; ++k)
      mbar_wait(full(k % kSmStages), (k / kSmStages) & 1);
  if (warp == 5 && lane == 0 && mmas > 0) mbar_wait(done((mmas - 1) % kSmStages), ((mmas - 1) / kSmStages) & 1);
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc_warp(tmem, kGrpTmemCols);
  }
}

// ---- host side ----

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// A [rows x 64] bf16 matrix of 128-B rows, copied as boxes of `box_rows` rows
// (8: one unit; 64: a whole indexer-key page) with the 128-byte swizzle.
static bool key_map(CUtensorMap* m, void* base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kIdxDim, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kIdxRowBytes};
  const cuuint32_t box[2] = {(cuuint32_t)kIdxDim, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t score_mma_set_attributes() {
  cudaError_t e = cudaFuncSetAttribute(score_mma_kernel<SRC_FLAT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kScoreMmaSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(score_mma_kernel<SRC_BLOCKKEYS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kScoreMmaSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(score_mma_kernel<SRC_POOL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kScoreMmaSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(score_mma_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGrpSmem);
  return e;
}

// bf16 keys: the same work split as the FFMA kernel (units per CTA chosen so
// that the batch fills three CTAs per SM), tiles of 16 units.
cudaError_t launch_score_mma(int src, const CacheView& c, const uint16_t* idx_q, const float* head_w,
                             const int32_t* q_seq, const int32_t* q_vis, const int32_t* pool, int nq,
                             int64_t max_units, int64_t stride, float* scores, float* block_max, int64_t bstride,
                             cudaStream_t st) {
  CUtensorMap m;
  const bool ok = src == SRC_BLOCKKEYS ? key_map(&m, c.bk, (uint64_t)c.n_pages * kBlocksPerPage, kBlock)
                 : src == SRC_FLAT     ? key_map(&m, c.idxk, (uint64_t)c.n_pages * kPageTokens, kPageTokens)
                                       : key_map(&m, c.idxk, (uint64_t)c.n_pages * kPageTokens, kBlock);
  if (!ok) return cudaErrorInvalidValue;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (src == SRC_FLAT && block_max == nullptr && nq >= 2 * kGrp) {
    // groups of 16 queries (two CTAs per SM)
    const int ngroups = (nq + kGrp - 1) / kGrp;
    int64_t per_group = ((int64_t)2 * sms) / ngroups;
    if (per_group < 1) per_group = 1;
    int64_t gupc = (max_units + per_group - 1) / per_group;
    gupc = (gupc + kTileUnits - 1) / kTileUnits * kTileUnits;
    if (gupc > kSmUnitsPerCta) gupc = kSmUnitsPerCta;
    if (gupc < kTileUnits) gupc = kTileUnits;
    const dim3 ggrid((unsigned)((max_units + gupc - 1) / gupc), (unsigned)ngroups);
    if (ggrid.x == 0) return cudaSuccess;
    launch_pdl(score_mma_group_kernel, ggrid, kSmThreads, kGrpSmem, st, m, c, idx_q, head_w, q_seq, q_vis, nq,
               max_units, stride, (int)gupc, scores);
    return cudaGetLastError();
  }
  int64_t per_query = nq > 0 ? ((int64_t)3 * sms) / nq : 1;
  if (per_query < 1) per_query = 1;
  int64_t upc = (max_units + per_query - 1) / per_query;
  upc = (upc + kTileUnits - 1) / kTileUnits * kTileUnits;
  if (upc > kSmUnitsPerCta) upc = kSmUnitsPerCta;
  if (upc < kTileUnits) upc = kTileUnits;
  dim3 grid((unsigned)((max_units + upc - 1) / upc), (unsigned)nq);
  if (grid.x == 0 || nq == 0) return cudaSuccess;
  if (src == SRC_FLAT)
    launch_pdl(score_mma_kernel<SRC_FLAT>, grid, kSmThreads, kScoreMmaSmem, st, m, c, idx_q, head_w, q_seq, q_vis, pool,
                                                                        max_units, stride, (int)upc, scores,
                                                                        block_max, bstride);
  else if (src == SRC_BLOCKKEYS)
    launch_pdl(score_mma_kernel<SRC_BLOCKKEYS>, grid, kSmThreads, kScoreMmaSmem, st, m, c, idx_q, head_w, q_seq, q_vis,
                                                                             pool, max_units, stride, (int)upc,
                                                                             scores, nullptr, 0);
  else
    launch_pdl(score_mma_kernel<SRC_POOL>, grid, kSmThreads, kScoreMmaSmem, st, m, c, idx_q, head_w, q_seq, q_vis, pool,
                                                                        max_units, stride, (int)upc, scores,
                                                                        nullptr, 0);
  return cudaGetLastError();
}

}  // namespace csa2
