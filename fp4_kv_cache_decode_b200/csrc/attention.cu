// CSA2 sparse attention over the FP4 cache on the 5th-generation tensor cores.
//
// A query attends over its selected positions joined with the 128-token
// sliding window (agentnet.co.il, "דיפסיק משיקה את V4.1-פלאש ...", sections
// "CSA2: דחיסה לאורך ציר השכבות" and "ארכיטקטורה שחותכת בחצי את הפריפיל").
// The selection is ascending, so the selected positions below the window
// start form a prefix of the index row and the attended list is
//   rows [0, n_sel)           = idx[0 .. n_sel)      (positions < w0)
//   rows [n_sel, n_sel + W')  = w0 .. v-1            (the window)
// with every position listed once.
//
// Work split: one CTA per (query, 128-row tile) -- at most 640 rows, so 5
// tiles -- followed by a combine kernel that merges the tiles' (m, l, O)
// with the usual log-sum-exp rule.  Per CTA (512 threads, one CTA per SM):
//   1. gather the tile's 288-B FP4 rows (16 lanes per row, coalesced) and
//      decode them to bf16 straight into shared memory in the UMMA 128-byte-swizzle K-major layout
//      (K^ [128 rows x 512 channels]); every E2M1 x E4M3 product is exact in
//      bf16 (byte-permute table lookup of the E2M1 magnitude, then one
//      bf16x2 multiply by the group scale);
//   2. copy the query [H x 512] (heads padded to 64 with zeros) into the
//      same layout;
//   3. one thread issues 32 tcgen05.mma (M=128 rows, N=64 heads, K=16):
//      S^T = K^ . Q^T accumulates in TMEM columns [0, 64);
//   4. each thread reads one row's 32 logits (tcgen05.ld), the tile-local
//      softmax max and sum per head are reduced across the 128 rows
//      (reduce-scatter shuffles + shared memory), and P^T is written as bf16
//      in the MN-major swizzled layout;
//   5. 32 more MMAs compute O^T = V^T . P^T (V = K^, read MN-major from the
//      same shared-memory bytes) into TMEM columns [64, 320);
//   6. O^T is read back (tcgen05.ld) and written with (m, l) to the workspace.
// MMA completion is tracked with tcgen05.commit on an mbarrier; every wait is
// bounded and reports CSA2_DEVERR_TIMEOUT instead of hanging.
#include "common.cuh"

namespace csa2 {

constexpr int kTile = 128;                          // attended rows per CTA (MMA M)
constexpr int kSplits = kMaxRows / kTile;           // 5
constexpr int kHeadsMma = 64;                       // MMA N: heads, padded
constexpr int kAttnThreads = 512;
constexpr uint32_t kKhBytes = 8u * kTile * 128u;    // 8 channel blocks x 128 rows x 128 B
constexpr uint32_t kQsBytes = 8u * kHeadsMma * 128u;
constexpr uint32_t kPsBytes = kTile * 128u;         // 128 rows x 64 heads x bf16
constexpr uint32_t kOffKh = 0;
constexpr uint32_t kOffQs = kOffKh + kKhBytes;
constexpr uint32_t kOffPs = kOffQs + kQsBytes;
constexpr uint32_t kOffRed = kOffPs + kPsBytes;     // float [2][4][64]
constexpr uint32_t kOffFin = kOffRed + 2048;        // float mfin[64], lfin[64]
constexpr uint32_t kOffPos = kOffFin + 512;         // int32 pos[128]
constexpr uint32_t kOffIdx = kOffPos + 512;         // int32 idx row [512]
constexpr uint32_t kOffRowp = kOffIdx + 2048;       // row base pointers [128]
constexpr uint32_t kOffMisc = kOffRowp + 1024;      // mbarrier, tmem base, n_sel
constexpr uint32_t kAttnSmem = kOffMisc + 64 + 1024;   // + slack for 1024-B alignment
constexpr uint32_t kTmemCols = 512;                 // S^T 64 + O^T 4 x 64 = 320, rounded up

// Instruction descriptors for tcgen05.mma kind::f16: D fp32 (bits 4-5 = 1),
// A and B bf16 (bits 7-9 = 1, 10-12 = 1), N>>3 at bit 17, M>>4 at bit 24;
// bit 15 / 16 = A / B are MN-major.
constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) |
                              ((uint32_t)(kHeadsMma >> 3) << 17) | ((uint32_t)(kTile >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescQK | (1u << 15) | (1u << 16);

constexpr uint32_t kWaitLimit = 1u << 24;

// Shared-memory matrix descriptor: start address, leading and stride byte
// offsets (16-B units), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
               : "memory");
}

__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(mbar), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 32 consecutive fp32 TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(d) : "f"(lo), "f"(hi));
  return d;
}

// Four E2M1 codes (16 bits, channel i in bits 4i..4i+3) -> two bf16x2 words of
// the unscaled values.  The 8 magnitudes' bf16 bytes are byte-permute tables:
// low bytes {00,00,80,C0,00,40,80,C0}, high bytes {00,3F,3F,3F,40,40,40,40}
// for 0, .5, 1, 1.5, 2, 3, 4, 6; the code's bit 3 becomes the bf16 sign.
// The four sign bits (code bits 3, 7, 11, 15) are moved to bit 7 of the
// matching high byte via the byte pattern [b0, b0, b1, b1] of the codes.
__device__ __forceinline__ void e2m1x4_to_bf16(uint32_t c16, uint32_t& w0, uint32_t& w1) {
  const uint32_t sel = c16 & 0x7777u;
  const uint32_t lo = __byte_perm(0xC0800000u, 0xC0804000u, sel);
  const uint32_t dup = __byte_perm(c16, 0u, 0x1100);
  const uint32_t hi = __byte_perm(0x3F3F3F00u, 0x40404040u, sel) | (dup & 0x80008000u) |
                      ((dup << 4) & 0x00800080u);
  w0 = __byte_perm(lo, hi, 0x5140);
  w1 = __byte_perm(lo, hi, 0x7362);
}

// 8 decoded channels (one 16-B chunk): codes word (4 bytes) x scale (bf16x2).
__device__ __forceinline__ uint4 decode8(uint32_t codes, uint32_t scale2) {
  uint4 o;
  uint32_t a, b;
  e2m1x4_to_bf16(codes & 0xFFFFu, a, b);
  o.x = mul_bf16x2(a, scale2);
  o.y = mul_bf16x2(b, scale2);
  e2m1x4_to_bf16(codes >> 16, a, b);
  o.z = mul_bf16x2(a, scale2);
  o.w = mul_bf16x2(b, scale2);
  return o;
}

// Lane l ends up with op over the 32 lanes of element l of v (31 shuffles).
template <bool kMax>
__device__ __forceinline__ float reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = up ? v[i] : v[i + w];
      const float keep = up ? v[i + w] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, w);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  return v[0];
}

__global__ void __launch_bounds__(kAttnThreads, 1)
attn_tile_kernel(CacheView c, const uint16_t* __restrict__ q, int H, float sm_scale,
                 const int32_t* __restrict__ q_seq, const int32_t* __restrict__ q_vis,
                 const int32_t* __restrict__ idx, float* __restrict__ part_o,
                 float2* __restrict__ part_ml) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw_s = (uint32_t)__cvta_generic_to_shared(smem_raw);
  const uint32_t sb = (raw_s + 1023u) & ~1023u;            // 1024-B aligned base (swizzle atoms)
  uint8_t* const sp = smem_raw + (sb - raw_s);
  float* const red = reinterpret_cast<float*>(sp + kOffRed);       // [2][4][64]
  float* const mfin = reinterpret_cast<float*>(sp + kOffFin);
  float* const lfin = mfin + 64;
  int32_t* const pos_s = reinterpret_cast<int32_t*>(sp + kOffPos);
  uint32_t* const misc = reinterpret_cast<uint32_t*>(sp + kOffMisc);  // [0..1] mbar, [2] tmem, [3] n_sel
  const uint32_t mbar = sb + kOffMisc;

  const int split = blockIdx.x;
  const int r = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int seq = q_seq[r];
  const int64_t v = q_vis ? (int64_t)q_vis[r] : (int64_t)seq_len_of(c, seq);
  const int64_t w0 = v > kWindow ? v - kWindow : 0;
  const int32_t* idx_row = idx + (int64_t)r * kTopK;
  float2* ml = part_ml + ((int64_t)r * kSplits + split) * H;

  // query -> Q tile (K-major, 128-B swizzle), asynchronous: head h, channel block kb, chunk j
  {
    const uint4* qsrc = reinterpret_cast<const uint4*>(q + (int64_t)r * H * kD);
#pragma unroll 4
    for (int e = tid; e < kHeadsMma * (kD / 8); e += kAttnThreads) {
      const int h = e >> 6, c16 = e & 63, kb = c16 >> 3, j = c16 & 7;
      const uint32_t off = kOffQs + kb * (kHeadsMma * 128u) + (h >> 3) * 1024u + (h & 7) * 128u +
                           ((j ^ (h & 7)) << 4);
      if (h < H) cp_async16(sb + off, qsrc + (h * (kD / 8) + c16));
      else *reinterpret_cast<uint4*>(sp + off) = make_uint4(0, 0, 0, 0);
    }
  }
  // selected positions below the window (a prefix of the ascending row)
  int32_t* const idx_s = reinterpret_cast<int32_t*>(sp + kOffIdx);
  if (tid == 0) misc[3] = 0;
  const int32_t e0 = idx_row[tid];    // kTopK == kAttnThreads
  idx_s[tid] = e0;
  __syncthreads();
  {
    int cnt = 0;
    if (e0 >= v) raise_error(c.err, CSA2_DEVERR_POS);
    cnt += (e0 >= 0 && e0 < w0) ? 1 : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) atomicAdd(&misc[3], (uint32_t)cnt);
  }
  __syncthreads();
  const int n_sel = (int)misc[3];
  const int64_t n_rows = n_sel + (v - w0);
  const int64_t row0 = (int64_t)split * kTile;
  if (row0 >= n_rows) {   // empty split: no TMEM is touched
    for (int h = tid; h < H; h += kAttnThreads) ml[h] = make_float2(-INFINITY, 0.0f);
    cp_async_wait_all();
    return;
  }
  const int rows = (int)(n_rows - row0 < kTile ? n_rows - row0 : kTile);

  // TMEM allocation (warp 0) and the MMA-completion mbarrier
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sb + kOffMisc + 8),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mbar));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  const uint8_t** const rowp = reinterpret_cast<const uint8_t**>(sp + kOffRowp);
  if (tid < kTile) {
    const int64_t i = row0 + tid;
    const int32_t p = tid < rows ? (i < n_sel ? idx_s[i] : (int32_t)(w0 + (i - n_sel))) : -1;
    pos_s[tid] = p;
    const uint8_t* rp = nullptr;
    if (p >= 0) {
      const int64_t pg = page_of(c, seq, p);
      if (pg >= 0) rp = c.kv + pg * kPageBytes + (p & (kPageTokens - 1)) * kRowBytes;
    }
    rowp[tid] = rp;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[2];

  // gather + decode: 16 lanes per row, lane piece p = 16 B of codes (channels
  // 32p .. 32p+31) plus its two scale bytes; a warp loads two rows per
  // instruction; 4 rounds of 32 rows.  All loads are issued before decoding.
  {
    const int piece = tid & 15;
    const int rsub = tid >> 4;                  // 0..31
    uint4 cw[4];
    uint32_t sw[4];
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const uint8_t* rp = rowp[rsub + 32 * it];
      if (rp) {
        cw[it] = __ldg(reinterpret_cast<const uint4*>(rp + piece * 16));
        sw[it] = __ldg(reinterpret_cast<const unsigned short*>(rp + kCodeBytes + piece * 2));
      } else {
        cw[it] = make_uint4(0, 0, 0, 0);
        sw[it] = 0;
      }
    }
    const int kb = piece >> 1;                  // 64-channel block
    const int half = piece & 1;                 // chunks 0-3 or 4-7 of the block's 128-B row
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int t = rsub + 32 * it;
      const bool have = rowp[t] != nullptr;
      const uint32_t base = kOffKh + kb * (kTile * 128u) + (t >> 3) * 1024u + (t & 7) * 128u;
      const uint32_t sb0 = __float_as_uint(e4m3_pos_value(sw[it] & 0x7Fu)) >> 16;
      const uint32_t sb1 = __float_as_uint(e4m3_pos_value((sw[it] >> 8) & 0x7Fu)) >> 16;
      const uint32_t s20 = sb0 | (sb0 << 16), s21 = sb1 | (sb1 << 16);
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = (jj + kb) & 3;            // rotate the store order across lanes (bank spread)
        const uint32_t cj = j == 0 ? cw[it].x : j == 1 ? cw[it].y : j == 2 ? cw[it].z : cw[it].w;
        const uint4 val = have ? decode8(cj, j < 2 ? s20 : s21) : make_uint4(0, 0, 0, 0);
        const int chunk = half * 4 + j;
        *reinterpret_cast<uint4*>(sp + base + ((chunk ^ (t & 7)) << 4)) = val;
      }
    }
  }
  cp_async_wait_all();
  fence_async_smem();
  __syncthreads();

  bool ok = true;
  // S^T = K^ . Q^T : M = 128 rows, N = 64 heads, K = 512 channels in 32 steps
  if (tid == 0) {
    tc_fence_after();
#pragma unroll 1
    for (int kb = 0; kb < 8; ++kb) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t a = smem_desc(sb + kOffKh + kb * (kTile * 128u) + ks * 32u, 16u, 1024u);
        const uint64_t b = smem_desc(sb + kOffQs + kb * (kHeadsMma * 128u) + ks * 32u, 16u, 1024u);
        mma_bf16(tmem, a, b, kIdescQK, (kb | ks) ? 1u : 0u);
      }
    }
    mma_commit(mbar);
  }
  if (!mbar_wait(mbar, 0)) ok = false;
  tc_fence_after();

  // softmax on warps 0..7: warp -> (TMEM lane quarter q4, head half hh)
  const bool smx = warp < 8;
  const int q4 = warp & 3, hh = (warp >> 2) & 1;
  const int t = q4 * 32 + lane;                 // this thread's attended row (TMEM lane)
  const bool valid = t < rows;
  float s[32], w[32];
  if (smx) {
    if (__all_sync(0xffffffffu, ok)) {
      tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + hh * 32, s);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) s[i] = 0.0f;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      s[i] = valid ? s[i] * sm_scale : -INFINITY;
      w[i] = s[i];
    }
    red[(0 * 4 + q4) * 64 + hh * 32 + lane] = reduce_scatter32<true>(w, lane);
  }
  __syncthreads();
  if (tid < 64) {
    const float* rm = red + tid;
    mfin[tid] = fmaxf(fmaxf(rm[0], rm[64]), fmaxf(rm[128], rm[192]));
  }
  __syncthreads();
  if (smx) {
    constexpr float kLog2e = 1.4426950408889634f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float m = mfin[hh * 32 + i];
      s[i] = valid ? exp2f((s[i] - m) * kLog2e) : 0.0f;
      w[i] = s[i];
    }
    red[(1 * 4 + q4) * 64 + hh * 32 + lane] = reduce_scatter32<false>(w, lane);
    // P^T (MN-major, 128-B swizzle): row t, heads hh*32 .. hh*32+31 = chunks 4hh .. 4hh+3
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint4 pk;
      pk.x = pack_bf16x2(s[8 * j + 0], s[8 * j + 1]);
      pk.y = pack_bf16x2(s[8 * j + 2], s[8 * j + 3]);
      pk.z = pack_bf16x2(s[8 * j + 4], s[8 * j + 5]);
      pk.w = pack_bf16x2(s[8 * j + 6], s[8 * j + 7]);
      const int cj = hh * 4 + j;
      *reinterpret_cast<uint4*>(sp + kOffPs + (t >> 3) * 1024u + (t & 7) * 128u + ((cj ^ (t & 7)) << 4)) = pk;
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid < 64) {
    const float* rs = red + 256 + tid;
    lfin[tid] = (rs[0] + rs[64]) + (rs[128] + rs[192]);
    if (tid < H) ml[tid] = make_float2(mfin[tid], lfin[tid]);
  }

  // O^T = V^T . P^T : 4 channel tiles (M = 128), N = 64 heads, K = 128 rows in 8 steps
  if (tid == 0) {
    tc_fence_after();
#pragma unroll 1
    for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t a = smem_desc(sb + kOffKh + (2 * mt) * (kTile * 128u) + ks * 2048u, kTile * 128u, 1024u);
        const uint64_t b = smem_desc(sb + kOffPs + ks * 2048u, 8192u, 1024u);
        mma_bf16(tmem + 64 + 64 * mt, a, b, kIdescPV, ks ? 1u : 0u);
      }
    }
    mma_commit(mbar);
  }
  if (!mbar_wait(mbar, 1)) ok = false;
  tc_fence_after();
  if (__all_sync(0xffffffffu, ok)) {
    float* o = part_o + (((int64_t)r * kSplits + split) * H) * kD;
    const int eq4 = warp & 3;                     // TMEM lane quarter of this warp
#pragma unroll 1
    for (int pr = warp >> 2; pr < 8; pr += kAttnThreads / 128) {   // (tile, half) pairs
      const int mt = pr >> 1, half = pr & 1;
      if (half * 32 >= H) continue;
      const int ch = mt * 128 + eq4 * 32 + lane;
      float ov[32];
      tmem_ld32(tmem + ((uint32_t)(eq4 * 32) << 16) + 64 + 64 * mt + 32 * half, ov);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int h = half * 32 + i;
        if (h < H) o[(int64_t)h * kD + ch] = ov[i];
      }
    }
  }
  if (!ok) {
    if (tid == 0) raise_error(c.err, CSA2_DEVERR_TIMEOUT);
    mbar_wait(mbar, 1);   // give in-flight MMAs a second bounded chance before freeing TMEM
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// Merge the tiles of each (query, head): out = sum_j e^(m_j-M) O_j / sum_j e^(m_j-M) l_j.
// CTA = (query, 4 heads); thread = 8 channels of one head.
__global__ void __launch_bounds__(256) attn_combine_kernel(int H, const float* __restrict__ part_o,
                                                           const float2* __restrict__ part_ml,
                                                           uint16_t* __restrict__ out) {
  const int r = blockIdx.y;
  const int h = blockIdx.x * 4 + (threadIdx.x >> 6);
  const int c8 = (threadIdx.x & 63) * 8;
  if (h >= H) return;
  float M = -INFINITY;
  float2 mls[kSplits];
#pragma unroll
  for (int j = 0; j < kSplits; ++j) {
    mls[j] = part_ml[((int64_t)r * kSplits + j) * H + h];
    if (mls[j].y > 0.0f) M = fmaxf(M, mls[j].x);
  }
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float den = 0.0f;
  if (M != -INFINITY) {
#pragma unroll
    for (int j = 0; j < kSplits; ++j) {
      if (!(mls[j].y > 0.0f)) continue;
      const float wgt = exp2f((mls[j].x - M) * 1.4426950408889634f);
      den = fmaf(wgt, mls[j].y, den);
      const float4* src = reinterpret_cast<const float4*>(part_o + (((int64_t)r * kSplits + j) * H + h) * kD + c8);
      const float4 a = src[0], b = src[1];
      acc[0] = fmaf(wgt, a.x, acc[0]); acc[1] = fmaf(wgt, a.y, acc[1]);
      acc[2] = fmaf(wgt, a.z, acc[2]); acc[3] = fmaf(wgt, a.w, acc[3]);
      acc[4] = fmaf(wgt, b.x, acc[4]); acc[5] = fmaf(wgt, b.y, acc[5]);
      acc[6] = fmaf(wgt, b.z, acc[6]); acc[7] = fmaf(wgt, b.w, acc[7]);
    }
  }
  const float inv = den > 0.0f ? 1.0f / den : 0.0f;
  uint4 o;
  o.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  o.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  o.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  o.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(out + ((int64_t)r * H + h) * kD + c8) = o;
}

}  // namespace csa2

// ---- launchers used by api.cu ----
namespace csa2 {

size_t attn_workspace_bytes(int nq, int H) {
  const size_t o = (size_t)nq * kSplits * H * kD * sizeof(float);
  const size_t ml = (size_t)nq * kSplits * H * sizeof(float2);
  return o + ml + 256;
}

cudaError_t attention_set_attributes() {
  return cudaFuncSetAttribute(attn_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kAttnSmem);
}

cudaError_t launch_attention(const CacheView& c, const uint16_t* q, int H, float sm_scale,
                             const int32_t* q_seq, const int32_t* q_vis, const int32_t* idx, int nq,
                             uint16_t* out, void* ws, cudaStream_t st) {
  if (nq == 0) return cudaSuccess;
  if (H % 16 != 0 || H < 16 || H > kHeadsMma) return cudaErrorInvalidValue;
  float* part_o = reinterpret_cast<float*>(ws);
  float2* part_ml = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(ws) +
                                              (size_t)nq * kSplits * H * kD * sizeof(float));
  attn_tile_kernel<<<dim3(kSplits, nq), kAttnThreads, kAttnSmem, st>>>(c, q, H, sm_scale, q_seq, q_vis,
                                                                       idx, part_o, part_ml);
  attn_combine_kernel<<<dim3((H + 3) / 4, nq), 256, 0, st>>>(H, part_o, part_ml, out);
  return cudaGetLastError();
}

}  // namespace csa2
