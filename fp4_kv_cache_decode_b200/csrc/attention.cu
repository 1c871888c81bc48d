// CSA2 sparse attention over the FP4 cache: split-K partials + LSE combine.
//
// A query attends over its selected positions joined with the 128-token
// sliding window (agentnet.co.il, "דיפסיק משיקה את V4.1-פלאש ...", sections
// "CSA2: דחיסה לאורך ציר השכבות" and "ארכיטקטורה שחותכת בחצי את הפריפיל").
// Because the selection is ascending, the selected positions below the
// window start form a prefix of the index row, so the attended list is
//   rows [0, n_sel)          = idx[0 .. n_sel)            (positions < w0)
//   rows [n_sel, n_sel + W') = w0 .. v-1                  (the window)
// with every position listed once.  The list is cut into splits of kSplitRows
// rows; each CTA gathers its split's 288-B rows, decodes them to bf16 in
// shared memory (exact: every E2M1 x E4M3 product fits bf16), computes the
// split's logits, an exact split-local softmax (max m, sum l) and the
// unnormalised output O = sum p k, and writes (m, l, O) to the workspace.  The
// combine kernel merges the splits: out = sum_j e^(m_j-M) O_j / sum_j e^(m_j-M) l_j.
#include "common.cuh"

namespace csa2 {

constexpr int kSplitRows = 64;
constexpr int kSplits = kMaxRows / kSplitRows;      // 10
constexpr int kKStride = kD + 8;                    // padded bf16 row stride in smem
constexpr int kSStride = kSplitRows + 1;            // padded fp32 logit row stride

template <int H>
struct AttnSmem {
  uint16_t k[kSplitRows][kKStride];
  uint16_t q[H][kKStride];
  float s[H][kSStride];
  int32_t pos[kSplitRows];
  int32_t n_sel;
};

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float* f) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

template <int H>
__global__ void __launch_bounds__(256) attn_split_kernel(CacheView c, const uint16_t* __restrict__ q,
                                                         float sm_scale, const int32_t* __restrict__ q_seq,
                                                         const int32_t* __restrict__ q_vis,
                                                         const int32_t* __restrict__ idx,
                                                         float* __restrict__ part_o,
                                                         float2* __restrict__ part_ml) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  AttnSmem<H>& sm = *reinterpret_cast<AttnSmem<H>*>(smem_raw);
  const int split = blockIdx.x;
  const int r = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int seq = q_seq[r];
  const int64_t v = q_vis ? (int64_t)q_vis[r] : (int64_t)seq_len_of(c, seq);
  const int64_t w0 = v > kWindow ? v - kWindow : 0;
  const int32_t* idx_row = idx + (int64_t)r * kTopK;

  // selected positions below the window (a prefix of the ascending row)
  if (tid == 0) sm.n_sel = 0;
  __syncthreads();
  {
    int cnt = 0;
    for (int j = tid; j < kTopK; j += 256) {
      const int32_t e = idx_row[j];
      if (e >= v) raise_error(c.err, CSA2_DEVERR_POS);
      cnt += (e >= 0 && e < w0) ? 1 : 0;
    }
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 1);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 2);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 4);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 8);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 16);
    if (lane == 0) atomicAdd(&sm.n_sel, cnt);
  }
  __syncthreads();
  const int n_sel = sm.n_sel;
  const int64_t n_rows = n_sel + (v - w0);
  const int64_t row0 = (int64_t)split * kSplitRows;
  float2* ml = part_ml + ((int64_t)r * kSplits + split) * H;
  if (row0 >= n_rows) {
    for (int h = tid; h < H; h += 256) ml[h] = make_float2(-INFINITY, 0.0f);
    return;
  }
  const int rows = (int)(n_rows - row0 < kSplitRows ? n_rows - row0 : kSplitRows);

  if (tid < kSplitRows) {
    const int64_t i = row0 + tid;
    sm.pos[tid] = tid < rows ? (i < n_sel ? idx_row[i] : (int32_t)(w0 + (i - n_sel))) : -1;
  }
  // query rows -> smem
  {
    const uint4* qsrc = reinterpret_cast<const uint4*>(q + (int64_t)r * H * kD);
    for (int e = tid; e < H * (kD / 8); e += 256) {
      const int h = e / (kD / 8), c8 = e % (kD / 8);
      *reinterpret_cast<uint4*>(&sm.q[h][c8 * 8]) = __ldg(qsrc + e);
    }
  }
  __syncthreads();

  // gather + decode: warp per row, lane per scale group
  for (int t = warp; t < kSplitRows; t += 8) {
    uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
    const int32_t p = sm.pos[t];
    int64_t pg = -1;
    if (p >= 0) pg = page_of(c, seq, p);
    if (pg >= 0) {
      const uint8_t* row = c.kv + pg * kPageBytes + (p & (kPageTokens - 1)) * kRowBytes;
      const uint2 cw = reinterpret_cast<const uint2*>(row)[lane];
      const float s = e4m3_pos_value(row[kCodeBytes + lane] & 0x7Fu);
      uint32_t o[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t word = j < 4 ? cw.x : cw.y;
        const uint32_t c0 = (word >> ((j & 3) * 8)) & 0xFu;
        const uint32_t c1 = (word >> ((j & 3) * 8 + 4)) & 0xFu;
        float a = e2m1_mag(c0 & 7u) * s;
        float b = e2m1_mag(c1 & 7u) * s;
        if (c0 & 8u) a = -a;
        if (c1 & 8u) b = -b;
        o[j] = (uint32_t)f32_to_bf16_rne(a) | ((uint32_t)f32_to_bf16_rne(b) << 16);
      }
      lo = make_uint4(o[0], o[1], o[2], o[3]);
      hi = make_uint4(o[4], o[5], o[6], o[7]);
    }
    *reinterpret_cast<uint4*>(&sm.k[t][lane * 16]) = lo;
    *reinterpret_cast<uint4*>(&sm.k[t][lane * 16 + 8]) = hi;
  }
  __syncthreads();

  // logits: thread tile of 4 heads x 4 rows
  {
    const int hg = tid >> 4, tg = tid & 15;
    if (hg * 4 < H) {
      float acc[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
      for (int c8 = 0; c8 < kD; c8 += 8) {
        float qf[4][8], kf[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i) unpack_bf16x8(*reinterpret_cast<const uint4*>(&sm.q[hg * 4 + i][c8]), qf[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) unpack_bf16x8(*reinterpret_cast<const uint4*>(&sm.k[tg + 16 * j][c8]), kf[j]);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[i][j] = fmaf(qf[i][e], kf[j][e], acc[i][j]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int t = tg + 16 * j;
          sm.s[hg * 4 + i][t] = t < rows ? acc[i][j] * sm_scale : -INFINITY;
        }
    }
  }
  __syncthreads();

  // split-local softmax: warp per head, lane per two rows
  for (int h = warp; h < H; h += 8) {
    const float s0 = sm.s[h][lane], s1 = sm.s[h][lane + 32];
    float m = fmaxf(s0, s1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float p0 = lane < rows ? expf(s0 - m) : 0.0f;
    const float p1 = lane + 32 < rows ? expf(s1 - m) : 0.0f;
    float l = p0 + p1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    sm.s[h][lane] = p0;
    sm.s[h][lane + 32] = p1;
    if (lane == 0) ml[h] = make_float2(m, l);
  }
  __syncthreads();

  // O = P K: thread owns H/4 heads x 8 channels
  {
    constexpr int HPT = H / 4;
    const int hg = tid >> 6, cg = tid & 63;
    float acc[HPT][8];
#pragma unroll
    for (int i = 0; i < HPT; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[i][e] = 0.0f;
    for (int t = 0; t < rows; ++t) {
      float kf[8];
      unpack_bf16x8(*reinterpret_cast<const uint4*>(&sm.k[t][cg * 8]), kf);
#pragma unroll
      for (int i = 0; i < HPT; ++i) {
        const float p = sm.s[hg * HPT + i][t];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i][e] = fmaf(p, kf[e], acc[i][e]);
      }
    }
    float* o = part_o + (((int64_t)r * kSplits + split) * H) * kD;
#pragma unroll
    for (int i = 0; i < HPT; ++i) {
      float4* dst = reinterpret_cast<float4*>(o + (int64_t)(hg * HPT + i) * kD + cg * 8);
      dst[0] = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
      dst[1] = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
    }
  }
}

// Merge the splits of each (query, head): out = sum_j e^(m_j-M) O_j / sum_j e^(m_j-M) l_j.
__global__ void __launch_bounds__(256) attn_combine_kernel(int H, const float* __restrict__ part_o,
                                                           const float2* __restrict__ part_ml,
                                                           uint16_t* __restrict__ out) {
  const int r = blockIdx.x;
  for (int e = threadIdx.x; e < H * (kD / 8); e += 256) {
    const int h = e / (kD / 8), c8 = (e % (kD / 8)) * 8;
    float M = -INFINITY;
    for (int j = 0; j < kSplits; ++j) {
      const float2 ml = part_ml[((int64_t)r * kSplits + j) * H + h];
      if (ml.y > 0.0f) M = fmaxf(M, ml.x);
    }
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    float den = 0.0f;
    if (M != -INFINITY) {
      for (int j = 0; j < kSplits; ++j) {
        const float2 ml = part_ml[((int64_t)r * kSplits + j) * H + h];
        if (!(ml.y > 0.0f)) continue;
        const float wgt = expf(ml.x - M);
        den = fmaf(wgt, ml.y, den);
        const float4* src = reinterpret_cast<const float4*>(part_o + (((int64_t)r * kSplits + j) * H + h) * kD + c8);
        const float4 a = src[0], b = src[1];
        acc[0] = fmaf(wgt, a.x, acc[0]); acc[1] = fmaf(wgt, a.y, acc[1]);
        acc[2] = fmaf(wgt, a.z, acc[2]); acc[3] = fmaf(wgt, a.w, acc[3]);
        acc[4] = fmaf(wgt, b.x, acc[4]); acc[5] = fmaf(wgt, b.y, acc[5]);
        acc[6] = fmaf(wgt, b.z, acc[6]); acc[7] = fmaf(wgt, b.w, acc[7]);
      }
    }
    const float inv = den > 0.0f ? 1.0f / den : 0.0f;
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = (uint32_t)f32_to_bf16_rne(acc[2 * i] * inv) | ((uint32_t)f32_to_bf16_rne(acc[2 * i + 1] * inv) << 16);
    *reinterpret_cast<uint4*>(out + ((int64_t)r * H + h) * kD + c8) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace csa2

// ---- launchers used by api.cu ----
namespace csa2 {

size_t attn_workspace_bytes(int nq, int H) {
  const size_t o = (size_t)nq * kSplits * H * kD * sizeof(float);
  const size_t ml = (size_t)nq * kSplits * H * sizeof(float2);
  return o + ml + 256;
}

template <int H>
static cudaError_t set_attn_attr() {
  return cudaFuncSetAttribute(attn_split_kernel<H>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)sizeof(AttnSmem<H>));
}

cudaError_t attention_set_attributes() {
  cudaError_t e = set_attn_attr<16>();
  if (e == cudaSuccess) e = set_attn_attr<32>();
  if (e == cudaSuccess) e = set_attn_attr<48>();
  if (e == cudaSuccess) e = set_attn_attr<64>();
  return e;
}

cudaError_t launch_attention(const CacheView& c, const uint16_t* q, int H, float sm_scale,
                             const int32_t* q_seq, const int32_t* q_vis, const int32_t* idx, int nq,
                             uint16_t* out, void* ws, cudaStream_t st) {
  if (nq == 0) return cudaSuccess;
  float* part_o = reinterpret_cast<float*>(ws);
  float2* part_ml = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(ws) +
                                              (size_t)nq * kSplits * H * kD * sizeof(float));
  dim3 grid(kSplits, nq);
  switch (H) {
    case 16: attn_split_kernel<16><<<grid, 256, sizeof(AttnSmem<16>), st>>>(c, q, sm_scale, q_seq, q_vis, idx, part_o, part_ml); break;
    case 32: attn_split_kernel<32><<<grid, 256, sizeof(AttnSmem<32>), st>>>(c, q, sm_scale, q_seq, q_vis, idx, part_o, part_ml); break;
    case 48: attn_split_kernel<48><<<grid, 256, sizeof(AttnSmem<48>), st>>>(c, q, sm_scale, q_seq, q_vis, idx, part_o, part_ml); break;
    case 64: attn_split_kernel<64><<<grid, 256, sizeof(AttnSmem<64>), st>>>(c, q, sm_scale, q_seq, q_vis, idx, part_o, part_ml); break;
    default: return cudaErrorInvalidValue;
  }
  attn_combine_kernel<<<nq, 256, 0, st>>>(H, part_o, part_ml, out);
  return cudaGetLastError();
}

}  // namespace csa2
