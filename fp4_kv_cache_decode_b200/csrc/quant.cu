// FP4 main-KV encoder (csa2_kv_quant_append, csa2_swa_replay) and block keys.
//
// Codec: E2M1 codes with one E4M3 scale per 16 channels and no global scale
// (agentnet.co.il, "דיפסיק משיקה את V4.1-פלאש ...", section "קוונטיזציה ופריסה:
// FP4 ו-DRAM במקום SSD").  One warp encodes one 512-channel row: lane l owns
// scale group l (channels 16l..16l+15), so the group maximum needs no
// cross-lane traffic; the 32 lanes' 8-byte code words form the row's 256
// code bytes in one coalesced 256-B store, their scale bytes the 32-B tail.
//
// Rounding is decided exactly:
//  * scale: fp32 amax/6 (IEEE division) then the hardware's round-to-nearest-
//    even, saturating E4M3 conversion.  For inputs with at most 24 significant
//    bits the correctly rounded quotient can neither reach nor cross an E4M3
//    midpoint that the exact quotient does not, so this equals rounding the
//    exact amax/6;
//  * code: |x| compared with midpoint x scale for the 7 E2M1 midpoints; each
//    product has at most 7 significant bits and is exact in fp32, so this is
//    the exact nearest-even rounding of |x|/scale, saturating at 6.
#include <cuda_fp8.h>

#include "common.cuh"

namespace csa2 {

struct GroupCode {
  uint2 codes;    // 16 nibbles, channel 2j of the group in the low nibble of byte j
  uint32_t scale; // E4M3 byte
};

// Encode the 16 values of one scale group.
__device__ __forceinline__ GroupCode encode_group(const float (&x)[16]) {
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(x[j]));
  const float q = __fdiv_rn(amax, 6.0f);
  const uint32_t sb = (uint32_t)__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3) & 0x7Fu;
  const float s = e4m3_pos_value(sb);
  GroupCode g;
  g.scale = sb;
  uint32_t w[2] = {0u, 0u};
  if (s != 0.0f) {
    // midpoints of the E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}, scaled (exact)
    const float t0 = 0.25f * s, t1 = 0.75f * s, t2 = 1.25f * s, t3 = 1.75f * s;
    const float t4 = 2.5f * s, t5 = 3.5f * s, t6 = 5.0f * s;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float a = fabsf(x[j]);
      uint32_t below = (t0 < a) + (t1 < a) + (t2 < a) + (t3 < a) + (t4 < a) + (t5 < a) + (t6 < a);
      const bool tie = (a == t0) | (a == t1) | (a == t2) | (a == t3) | (a == t4) | (a == t5) |
                       (a == t6);
      below += (tie && (below & 1u)) ? 1u : 0u;
      const uint32_t code = below | ((__float_as_uint(x[j]) >> 31) << 3);
      w[j >> 3] |= code << ((j & 7) * 4);
    }
  }
  g.codes = make_uint2(w[0], w[1]);
  return g;
}

// Unpack 8 bf16 values from a 16-B word.
__device__ __forceinline__ void unpack8(const uint4& v, float* out) {
  out[0] = bf16_lo(v.x); out[1] = bf16_hi(v.x);
  out[2] = bf16_lo(v.y); out[3] = bf16_hi(v.y);
  out[4] = bf16_lo(v.z); out[5] = bf16_hi(v.z);
  out[6] = bf16_lo(v.w); out[7] = bf16_hi(v.w);
}

// One lane's share of an entry's source: scale group `lane` of the one or two
// (compress 1 or 2) consecutive bf16 rows of 512 at kv_src.  Loaded before the
// entry's position is known, so that these loads overlap the lookups.
struct SrcWords {
  uint4 a0, a1, b0, b1;
};

__device__ __forceinline__ SrcWords load_src_lane(int lane, const uint16_t* __restrict__ kv_src, int compress) {
  SrcWords w;
  const uint4* r0 = reinterpret_cast<const uint4*>(kv_src) + lane * 2;
  w.a0 = __ldg(r0);
  w.a1 = __ldg(r0 + 1);
  if (compress == 2) {
    const uint4* r1 = reinterpret_cast<const uint4*>(kv_src + kD) + lane * 2;
    w.b0 = __ldg(r1);
    w.b1 = __ldg(r1 + 1);
  } else {
    w.b0 = w.b1 = make_uint4(0, 0, 0, 0);
  }
  return w;
}

// The FP4 code of scale group `lane` of an entry (pair mean in fp32 at ratio 2).
__device__ __forceinline__ GroupCode encode_src_lane(const SrcWords& w, int compress) {
  float x[16];
  unpack8(w.a0, x);
  unpack8(w.a1, x + 8);
  if (compress == 2) {
    float y[16];
    unpack8(w.b0, y);
    unpack8(w.b1, y + 8);
#pragma unroll
    for (int j = 0; j < 16; ++j) x[j] = __fmul_rn(__fadd_rn(x[j], y[j]), 0.5f);
  }
  return encode_group(x);
}

// One warp: store a row's codes (256 B) and scales (32 B tail).
__device__ __forceinline__ void store_row_warp(uint8_t* row, int lane, const GroupCode& g) {
  reinterpret_cast<uint2*>(row)[lane] = g.codes;
  row[kCodeBytes + lane] = (uint8_t)g.scale;
}

// One warp: the stored indexer key of an entry (lane owns dims 2 lane, 2 lane + 1;
// pair mean rounded to bf16 at ratio 2).
__device__ __forceinline__ uint32_t idxk_src_warp(int lane, const uint16_t* __restrict__ idxk_src,
                                                  int compress) {
  uint32_t kw = __ldg(reinterpret_cast<const uint32_t*>(idxk_src) + lane);
  if (compress == 2) {
    const uint32_t kw2 = __ldg(reinterpret_cast<const uint32_t*>(idxk_src + kIdxDim) + lane);
    const float a = __fmul_rn(__fadd_rn(bf16_lo(kw), bf16_lo(kw2)), 0.5f);
    const float b = __fmul_rn(__fadd_rn(bf16_hi(kw), bf16_hi(kw2)), 0.5f);
    kw = (uint32_t)f32_to_bf16_rne(a) | ((uint32_t)f32_to_bf16_rne(b) << 16);
  }
  return kw;
}

// One warp: store an indexer key (lane holds dims 2 lane, 2 lane + 1 as bf16)
// as FP8 at slot `slot` of an FP8 key page: scale s = fl32(amax / 448), codes
// = E4M3(fl32(k / s)) rounded to nearest even with saturation at 448.
__device__ __forceinline__ void store_idxk_fp8(uint8_t* page, int slot, int lane, uint32_t kw) {
  const float a = bf16_lo(kw), b = bf16_hi(kw);
  float amax = fmaxf(fabsf(a), fabsf(b));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = __fdiv_rn(amax, 448.0f);
  uint16_t code = 0;
  if (s != 0.0f)
    code = (uint16_t)__nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(a, s), __fdiv_rn(b, s)), __NV_SATFINITE,
                                              __NV_E4M3);
  reinterpret_cast<uint16_t*>(page + slot * kIdx8RowBytes)[lane] = code;
  if (lane == 0) reinterpret_cast<float*>(page + kIdx8ScaleOff)[slot] = s;
}

// Slot of position pos of sequence seq in the sliding-window store.
__device__ __forceinline__ uint8_t* swa_row(const CacheView& c, int seq, int64_t pos) {
  return c.swa + ((int64_t)seq * kReplay + (pos & (kReplay - 1))) * kRowBytes;
}

// One warp: encode an entry into the cache row at (seq, pos) and store its
// indexer key; with a sliding-window store, an entry among the sequence's
// last 128 positions (pos >= len - 128) is also written to its slot there.
__device__ __forceinline__ void encode_entry_warp(const CacheView& c, int lane, const SrcWords& src,
                                                 const uint16_t* __restrict__ idxk_src,
                                                 int compress, int seq, int64_t pos, int64_t len) {
  const int64_t page = page_of(c, seq, pos);
  if (page < 0) return;
  const GroupCode g = encode_src_lane(src, compress);
  store_row_warp(c.kv + page * kPageBytes + (pos & (kPageTokens - 1)) * kRowBytes, lane, g);
  if (c.swa && pos >= len - kReplay) store_row_warp(swa_row(c, seq, pos), lane, g);
  const uint32_t kw = idxk_src_warp(lane, idxk_src, compress);
  if (c.idxk_fp8) {
    store_idxk_fp8(c.idxk + page * kIdx8PageBytes, (int)(pos & (kPageTokens - 1)), lane, kw);
  } else {
    uint8_t* krow = c.idxk + page * kIdxPageBytes + (pos & (kPageTokens - 1)) * kIdxRowBytes;
    reinterpret_cast<uint32_t*>(krow)[lane] = kw;
  }
}

// One warp: recompute the block key of block `blk` of sequence `seq` from the
// stored keys of its present tokens [8*blk, min(8*blk+8, len)) (FP8 keys
// through their dequantised values fl32(s x code)).
__device__ __forceinline__ void block_key_warp(const CacheView& c, int lane, int seq, int64_t blk,
                                               int64_t len) {
  const int64_t t0 = blk * kBlock;
  if (t0 >= len || t0 < 0) return;
  const int64_t page = page_of(c, seq, t0);
  if (page < 0) return;
  const int64_t t1 = min(t0 + kBlock, len);
  float a = 0.0f, b = 0.0f;
  if (c.idxk_fp8) {
    const uint8_t* kp = c.idxk + page * kIdx8PageBytes;
    for (int64_t t = t0; t < t1; ++t) {
      const int slot = (int)(t & (kPageTokens - 1));
      const uint32_t cw = reinterpret_cast<const uint16_t*>(kp + slot * kIdx8RowBytes)[lane];
      const float s = reinterpret_cast<const float*>(kp + kIdx8ScaleOff)[slot];
      const float2 v = e4m3x2_to_float2(cw);
      a = __fadd_rn(a, __fmul_rn(s, v.x));
      b = __fadd_rn(b, __fmul_rn(s, v.y));
    }
  } else {
    const uint8_t* kp = c.idxk + page * kIdxPageBytes;
    for (int64_t t = t0; t < t1; ++t) {
      const uint32_t w = reinterpret_cast<const uint32_t*>(kp + (t & (kPageTokens - 1)) * kIdxRowBytes)[lane];
      a = __fadd_rn(a, bf16_lo(w));
      b = __fadd_rn(b, bf16_hi(w));
    }
  }
  const float n = (float)(t1 - t0);
  const uint32_t out = (uint32_t)f32_to_bf16_rne(__fdiv_rn(a, n)) |
                       ((uint32_t)f32_to_bf16_rne(__fdiv_rn(b, n)) << 16);
  uint8_t* dst = c.bk + page * kBkPageBytes + (blk & (kBlocksPerPage - 1)) * kIdxRowBytes;
  reinterpret_cast<uint32_t*>(dst)[lane] = out;
}

constexpr int kWarpsPerCta = 8;

__global__ void __launch_bounds__(256) append_rows_kernel(CacheView c, const uint16_t* __restrict__ kv,
                                                          const uint16_t* __restrict__ idxk,
                                                          const int32_t* __restrict__ eseq,
                                                          const int32_t* __restrict__ epos, int n,
                                                          int compress) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (i >= n) return;
  const SrcWords src = load_src_lane(lane, kv + (int64_t)i * compress * kD, compress);
  const int seq = eseq[i];
  const int64_t pos = epos[i];
  if (seq < 0 || seq >= c.batch) {
    if (lane == 0) raise_error(c.err, CSA2_DEVERR_SEQ);
    return;
  }
  const int64_t len = c.seq_lens[seq];
  if (pos < 0 || pos >= len) {
    if (lane == 0) raise_error(c.err, CSA2_DEVERR_POS);
    return;
  }
  encode_entry_warp(c, lane, src, idxk + (int64_t)i * compress * kIdxDim, compress, seq, pos, len);
}

// Block keys of the blocks touched by an append.  Entry i recomputes its
// block unless entry i-1 touched the same block (the usual contiguous case);
// a block listed twice non-contiguously is recomputed twice to the same value.
__global__ void __launch_bounds__(256) append_block_keys_kernel(CacheView c,
                                                                const int32_t* __restrict__ eseq,
                                                                const int32_t* __restrict__ epos,
                                                                int n) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (i >= n) return;
  const int seq = eseq[i];
  const int64_t pos = epos[i];
  if (seq < 0 || seq >= c.batch || pos < 0) return;
  const int64_t len = c.seq_lens[seq];
  if (pos >= len) return;
  const int64_t blk = pos / kBlock;
  if (i > 0 && eseq[i - 1] == seq && epos[i - 1] >= 0 && epos[i - 1] / kBlock == blk) return;
  block_key_warp(c, lane, seq, blk, len);
}

// Replay: warp (b, r) handles entry r of the supplied last-128 block of seq b
// (raw rows [compress r, compress r + compress) of that block).  With a
// sliding-window store only its slot is rewritten; otherwise the cache row and
// the indexer key.
__global__ void __launch_bounds__(256) replay_rows_kernel(CacheView c, const uint16_t* __restrict__ kv_last,
                                                          const uint16_t* __restrict__ idxk_last,
                                                          const uint8_t* __restrict__ miss, int compress) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int r = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (r >= kReplay) return;
  const int64_t len = c.seq_lens[b];
  const int64_t nrep = miss[b] ? (len < kReplay ? len : (int64_t)kReplay) : (len > 0 ? 1 : 0);
  if (r < kReplay - nrep) return;
  const int64_t pos = len - kReplay + r;
  const int64_t row = ((int64_t)b * kReplay + r) * compress;
  // the source loads and the page lookup below are in flight together
  const SrcWords src = load_src_lane(lane, kv_last + row * kD, compress);
  if (c.swa) {
    store_row_warp(swa_row(c, b, pos), lane, encode_src_lane(src, compress));
    return;
  }
  encode_entry_warp(c, lane, src, idxk_last + row * kIdxDim, compress, b, pos, len);
}

// Replay block keys: warp (b, j) recomputes the j-th block touched in seq b.
__global__ void __launch_bounds__(256) replay_block_keys_kernel(CacheView c, const uint8_t* __restrict__ miss) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int j = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  const int64_t len = c.seq_lens[b];
  const int64_t nrep = miss[b] ? (len < kReplay ? len : (int64_t)kReplay) : (len > 0 ? 1 : 0);
  if (nrep == 0) return;
  const int64_t first = (len - nrep) / kBlock, last = (len - 1) / kBlock;
  if (first + j > last) return;
  block_key_warp(c, lane, b, first + j, len);
}

}  // namespace csa2

// ---- launchers used by api.cu ----
namespace csa2 {

cudaError_t launch_append(const CacheView& c, const uint16_t* kv, const uint16_t* idxk,
                          const int32_t* eseq, const int32_t* epos, int n, int compress,
                          cudaStream_t st) {
  const int grid = (n + kWarpsPerCta - 1) / kWarpsPerCta;
  launch_pdl(append_rows_kernel, grid, 256, 0, st, c, kv, idxk, eseq, epos, n, compress);
  launch_pdl(append_block_keys_kernel, grid, 256, 0, st, c, eseq, epos, n);
  return cudaGetLastError();
}

cudaError_t launch_replay(const CacheView& c, const uint16_t* kv_last, const uint16_t* idxk_last,
                          const uint8_t* miss, int compress, cudaStream_t st) {
  dim3 g1(kReplay / kWarpsPerCta, c.batch);
  launch_pdl(replay_rows_kernel, g1, 256, 0, st, c, kv_last, idxk_last, miss, compress);
  if (c.swa) return cudaGetLastError();   // the global cache's keys are untouched
  // a 128-token window touches at most 17 blocks of 8
  dim3 g2((kReplay / kBlock + 1 + kWarpsPerCta - 1) / kWarpsPerCta, c.batch);
  launch_pdl(replay_block_keys_kernel, g2, 256, 0, st, c, miss);
  return cudaGetLastError();
}

}  // namespace csa2
