// CSA2 sparse attention over the FP4 cache on the 5th-generation tensor cores.
//
// A query attends over its selected positions joined with the 128-token
// sliding window (agentnet.co.il, "דיפסיק משיקה את V4.1-פלאש ...", sections
// "CSA2: דחיסה לאורך ציר השכבות" and "ארכיטקטורה שחותכת בחצי את הפריפיל").
// The selection is ascending, so the selected positions below the window
// start form a prefix of the index row and the attended list is
//   rows [0, n_sel)           = idx[0 .. n_sel)      (positions < w0)
//   rows [n_sel, n_sel + W')  = w0 .. v-1            (the window)
// with every position listed once (at most 640 rows).
//
// Work split: a query's row list is cut into S contiguous ranges, one CTA
// each (S chosen so that the grid fills the GPU; S = 1 for large batches).
// A CTA walks its range in 64-row tiles through a warp-specialised pipeline:
//   * producer warps (8) gather the tile's 288-B FP4 rows (16 lanes per row,
//     coalesced) and decode them to bf16 straight into one of two shared-
//     memory buffers in the UMMA 128-byte-swizzle K-major layout; every
//     E2M1 x E4M3 product is exact in bf16 (byte-permute lookup of the E2M1
//     magnitude, one bf16x2 multiply by the group scale);
//   * one MMA thread issues S^T = K^ . Q^T (tcgen05.mma, M = 64 rows, N = 64
//     heads, K = 512) into one of two TMEM score buffers -- the next tile's
//     QK runs while the current tile's softmax does -- and, once P^T is
//     ready, O^T += V^T . P^T (M = 128 channels x 4, N = 64, K = 64) into a
//     TMEM accumulator that persists across the CTA's tiles (V = K^, read
//     MN-major from the same bytes);
//   * softmax warps (4, one per TMEM sub-partition) keep a running max m and
//     sum l per head (online softmax).  The max used for the exponentials is
//     only moved when a tile exceeds it by more than 8 (natural log), and
//     then O^T and l are rescaled in place, so exponentials stay <= e^8 and
//     the final O / l is exact up to rounding.
// With S = 1 the CTA writes the normalised bf16 output; otherwise it writes
// (m, l, O) and a combine kernel merges the S ranges (log-sum-exp).
// Hand-offs use mbarriers (tcgen05.commit for tensor-core completion); every
// wait is bounded and reports CSA2_DEVERR_TIMEOUT instead of hanging.
#include "common.cuh"

namespace csa2 {

constexpr int kRowTile = 64;                           // attended rows per pipeline step
constexpr int kMaxSplits = kMaxRows / kRowTile;        // 10
constexpr int kHeadsMma = 64;                          // MMA N: heads, padded
constexpr int kSoftmaxWarps = 4;                       // warps 0..3 (TMEM sub-partitions 0..3)
constexpr int kProducerWarps = 8;                      // warps 4..11
constexpr int kMmaWarp = kSoftmaxWarps + kProducerWarps;   // warp 12
constexpr int kPipeThreads = 32 * (kMmaWarp + 1);      // 416
constexpr int kProdThreads = 32 * kProducerWarps;      // 256
constexpr int kSmxThreads = 32 * kSoftmaxWarps;        // 128

constexpr uint32_t kQsBytes = 8u * kHeadsMma * 128u;   // 64 KiB: Q [64 heads x 512], 8 channel blocks
constexpr uint32_t kKtBytes = 8u * kRowTile * 128u;    // 64 KiB: K^ tile [64 rows x 512]
constexpr uint32_t kPtBytes = kRowTile * 128u;         // 8 KiB: P^T tile [64 rows x 64 heads]
constexpr uint32_t kOffQs = 0;
constexpr uint32_t kOffK = kOffQs + kQsBytes;          // two K^ buffers
constexpr uint32_t kOffP = kOffK + 2 * kKtBytes;       // two P^T buffers
constexpr uint32_t kOffRedM = kOffP + 2 * kPtBytes;    // float [4][64] tile max per warp
constexpr uint32_t kOffRedL = kOffRedM + 1024;         // float [4][64] tile sum per warp
constexpr uint32_t kOffRun = kOffRedL + 1024;          // float m_run[64], l_run[64], fac[64], m_tile[64]
constexpr uint32_t kOffRows = kOffRun + 1024;          // uint32 physical row ids [640]
constexpr uint32_t kOffBar = kOffRows + 4u * kMaxRows; // 8 mbarriers, TMEM base, counters
constexpr uint32_t kPipeSmem = kOffBar + 128 + 1024;   // + slack for 1024-B alignment
constexpr uint32_t kTmemCols = 512;                    // S^T 2 x 64 + O^T 4 x 64 = 384, rounded up
constexpr uint32_t kColO = 128;                        // first O^T column
constexpr uint32_t kNoRow = 0xFFFFFFFFu;
constexpr float kRescaleSlack = 8.0f;                  // natural-log headroom before the max moves

// Instruction descriptors for tcgen05.mma kind::f16: D fp32 (bits 4-5 = 1),
// A and B bf16 (bits 7-9 = 1, 10-12 = 1), N>>3 at bit 17, M>>4 at bit 24;
// bit 15 / 16 = A / B are MN-major.
constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) |
                              ((uint32_t)(kHeadsMma >> 3) << 17) | ((uint32_t)(kRowTile >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                              ((uint32_t)(kHeadsMma >> 3) << 17) | (8u << 24);


constexpr uint32_t kWaitLimit = 1u << 22;

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


__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}\n" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void smx_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kSmxThreads) : "memory"); }

// Barrier over the softmax warps that also ANDs a predicate across them, so
// that every softmax thread takes the same branch after a bounded wait.
__device__ __forceinline__ bool smx_all(bool p) {
  uint32_t res;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\tsetp.ne.b32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, 1, %2, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}\n"
      : "=r"(res)
      : "r"((uint32_t)p), "n"(kSmxThreads)
      : "memory");
  return res != 0;
}

// 32 consecutive fp32 TMEM columns from `v` into this thread's lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
      "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]),
      "f"(v[16]), "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]),
      "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}

// Over lanes 0..15 (and separately 16..31): lane l ends with op over the 16
// lanes of elements 4(l%16) .. 4(l%16)+3 of v[64] (60 shuffles).
template <bool kMax>
__device__ __forceinline__ void reduce_scatter16x64(float (&v)[64], int lane, float (&res)[4]) {
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < 4 * w; ++i) {
      const float send = up ? v[i] : v[i + 4 * w];
      const float keep = up ? v[i + 4 * w] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, w);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) res[e] = v[e];
}

__global__ void __launch_bounds__(kPipeThreads, 1)
attn_pipe_kernel(CacheView c, const uint16_t* __restrict__ q, int H, float sm_scale,
                 const int32_t* __restrict__ q_seq, const int32_t* __restrict__ q_vis,
                 const int32_t* __restrict__ idx, int nsplit, int range_rows,
                 uint16_t* __restrict__ out, float* __restrict__ part_o, float2* __restrict__ part_ml) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw_s = (uint32_t)__cvta_generic_to_shared(smem_raw);
  const uint32_t sb = (raw_s + 1023u) & ~1023u;            // 1024-B aligned base (swizzle atoms)
  uint8_t* const sp = smem_raw + (sb - raw_s);
  float* const red_m = reinterpret_cast<float*>(sp + kOffRedM);
  float* const red_l = reinterpret_cast<float*>(sp + kOffRedL);
  float* const m_run = reinterpret_cast<float*>(sp + kOffRun);
  float* const l_run = m_run + 64;
  float* const fac = m_run + 128;
  float* const m_tile = m_run + 192;
  uint32_t* const rows_s = reinterpret_cast<uint32_t*>(sp + kOffRows);
  uint32_t* const misc = reinterpret_cast<uint32_t*>(sp + kOffBar + 64);   // [0] tmem, [1] n_sel, [2] flags
  const uint32_t bar0 = sb + kOffBar;
  auto kfull = [&](int b) { return bar0 + 8u * b; };
  auto kempty = [&](int b) { return bar0 + 16u + 8u * b; };
  auto sfull = [&](int b) { return bar0 + 32u + 8u * b; };
  auto pfull = [&](int b) { return bar0 + 48u + 8u * b; };

  const int split = blockIdx.x;
  const int r = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int seq = q_seq[r];
  const int64_t v = q_vis ? (int64_t)q_vis[r] : (int64_t)seq_len_of(c, seq);
  const int64_t w0 = v > kWindow ? v - kWindow : 0;
  const int32_t* idx_row = idx + (int64_t)r * kTopK;

  // query -> Q (K-major, 128-B swizzle), asynchronous; heads >= H are zero
  {
    const uint4* qsrc = reinterpret_cast<const uint4*>(q + (int64_t)r * H * kD);
    for (int e = tid; e < kHeadsMma * (kD / 8); e += kPipeThreads) {
      const int h = e >> 6, c16 = e & 63, kb = c16 >> 3, j = c16 & 7;
      const uint32_t off = kOffQs + kb * (kHeadsMma * 128u) + (h >> 3) * 1024u + (h & 7) * 128u +
                           ((j ^ (h & 7)) << 4);
      if (h < H) cp_async16(sb + off, qsrc + (h * (kD / 8) + c16));
      else *reinterpret_cast<uint4*>(sp + off) = make_uint4(0, 0, 0, 0);
    }
  }
  // selected positions below the window (a prefix of the ascending row)
  if (tid == 0) {
    misc[1] = 0;
    misc[2] = 0;
    misc[3] = 0;   // last barrier the MMA thread committed to (0: none)
    misc[4] = 0;
  }
  __syncthreads();
  {
    int cnt = 0;
    for (int j = tid; j < kTopK; j += kPipeThreads) {
      const int32_t e = idx_row[j];
      if (e >= v) raise_error(c.err, CSA2_DEVERR_POS);
      cnt += (e >= 0 && e < w0) ? 1 : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0 && cnt) atomicAdd(&misc[1], (uint32_t)cnt);
  }
  __syncthreads();
  const int n_sel = (int)misc[1];
  const int64_t n_rows = n_sel + (v - w0);
  const int64_t rb = (int64_t)split * range_rows;
  const int64_t re = min(rb + (int64_t)range_rows, n_rows);
  if (rb >= re) {   // nothing to attend in this range: no TMEM is touched
    if (nsplit > 1) {
      float2* ml = part_ml + ((int64_t)r * nsplit + split) * H;
      for (int h = tid; h < H; h += kPipeThreads) ml[h] = make_float2(-INFINITY, 0.0f);
    } else {
      for (int e = tid; e < H * (kD / 8); e += kPipeThreads)
        reinterpret_cast<uint4*>(out + (int64_t)r * H * kD)[e] = make_uint4(0, 0, 0, 0);
    }
    cp_async_wait_all();
    return;
  }
  const int nrow = (int)(re - rb);
  const int nt = (nrow + kRowTile - 1) / kRowTile;

  // physical row ids of the range
  for (int i = tid; i < nrow; i += kPipeThreads) {
    const int64_t li = rb + i;
    const int32_t p = li < n_sel ? idx_row[li] : (int32_t)(w0 + (li - n_sel));
    uint32_t id = kNoRow;
    if (p >= 0) {
      const int64_t pg = page_of(c, seq, p);
      if (pg >= 0) id = (uint32_t)(pg * kPageTokens + (p & (kPageTokens - 1)));
    }
    rows_s[i] = id;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sb + kOffBar + 64),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(kfull(b), kProdThreads);
      mbar_init(kempty(b), 1);
      mbar_init(sfull(b), 1);
      mbar_init(pfull(b), kSmxThreads);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  cp_async_wait_all();
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  bool ok = true;

  if (warp >= kSoftmaxWarps && warp < kMmaWarp) {
    // ---------------- producers: gather + decode ----------------
    const int ptid = tid - kSmxThreads;
    const int piece = ptid & 15, rsub = ptid >> 4;       // 16 lanes per row, 16 rows per round
    const int kb = piece >> 1, half = piece & 1;
    for (int t = 0; t < nt && ok; ++t) {
      const int b = t & 1;
      if (t >= 2 && !mbar_wait(kempty(b), ((t - 2) >> 1) & 1)) { ok = false; break; }
      uint4 cw[4];
      uint32_t sw[4];
      bool have[4];
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int row = rsub + 16 * it;
        const int li = t * kRowTile + row;
        const uint32_t id = li < nrow ? rows_s[li] : kNoRow;
        have[it] = id != kNoRow;
        if (have[it]) {
          const uint8_t* rp = c.kv + (int64_t)id * kRowBytes;
          cw[it] = __ldg(reinterpret_cast<const uint4*>(rp + piece * 16));
          sw[it] = __ldg(reinterpret_cast<const unsigned short*>(rp + kCodeBytes + piece * 2));
        } else {
          cw[it] = make_uint4(0, 0, 0, 0);
          sw[it] = 0;
        }
      }
      const uint32_t kbase = kOffK + b * kKtBytes + kb * (kRowTile * 128u);
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int row = rsub + 16 * it;
        const uint32_t base = kbase + (row >> 3) * 1024u + (row & 7) * 128u;
        const uint32_t sb0 = __float_as_uint(e4m3_pos_value(sw[it] & 0x7Fu)) >> 16;
        const uint32_t sb1 = __float_as_uint(e4m3_pos_value((sw[it] >> 8) & 0x7Fu)) >> 16;
        const uint32_t s20 = sb0 | (sb0 << 16), s21 = sb1 | (sb1 << 16);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = (jj + kb) & 3;                   // rotate the store order (bank spread)
          const uint32_t cj = j == 0 ? cw[it].x : j == 1 ? cw[it].y : j == 2 ? cw[it].z : cw[it].w;
          const uint4 val = have[it] ? decode8(cj, j < 2 ? s20 : s21) : make_uint4(0, 0, 0, 0);
          const int chunk = half * 4 + j;
          *reinterpret_cast<uint4*>(sp + base + ((chunk ^ (row & 7)) << 4)) = val;
        }
      }
      fence_async_smem();
      mbar_arrive(kfull(b));
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issue (one thread) ----------------
    if (lane == 0) {
      auto issue_qk = [&](int t) -> bool {
        const int b = t & 1;
        if (!mbar_wait(kfull(b), (t >> 1) & 1)) return false;
        tc_fence_after();
#pragma unroll 1
        for (int kb = 0; kb < 8; ++kb) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t a = smem_desc(sb + kOffK + b * kKtBytes + kb * (kRowTile * 128u) + ks * 32u, 16u, 1024u);
            const uint64_t bq = smem_desc(sb + kOffQs + kb * (kHeadsMma * 128u) + ks * 32u, 16u, 1024u);
            mma_bf16(tmem + 64u * b, a, bq, kIdescQK, (kb | ks) ? 1u : 0u);
          }
        }
        mma_commit(sfull(b));
        misc[3] = sfull(b);
        misc[4] = (t >> 1) & 1;
        return true;
      };
      ok = issue_qk(0);
      for (int t = 0; t < nt && ok; ++t) {
        if (t + 1 < nt && !issue_qk(t + 1)) { ok = false; break; }
        const int b = t & 1;
        if (!mbar_wait(pfull(b), (t >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t a = smem_desc(sb + kOffK + b * kKtBytes + (2 * mt) * (kRowTile * 128u) + ks * 2048u,
                                         kRowTile * 128u, 1024u);
            const uint64_t bp = smem_desc(sb + kOffP + b * kPtBytes + ks * 2048u, 8192u, 1024u);
            mma_bf16(tmem + kColO + 64u * mt, a, bp, kIdescPV, (t > 0 || ks > 0) ? 1u : 0u);
          }
        }
        mma_commit(kempty(b));
        misc[3] = kempty(b);
        misc[4] = (t >> 1) & 1;
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax warps 0..3 ----------------
    const int sw_ = warp;                             // TMEM sub-partition == warp
    const int hl = lane & 15;
    const bool lo_half = lane < 16;
    constexpr float kLog2e = 1.4426950408889634f;
    for (int t = 0; t < nt && ok; ++t) {
      const int b = t & 1;
      if (!smx_all(mbar_wait(sfull(b), (t >> 1) & 1))) { ok = false; break; }
      tc_fence_after();
      const int row = 16 * sw_ + hl;                  // tile row held by lanes 0..15
      const bool valid = lo_half && (t * kRowTile + row) < nrow;
      float s[64], w[64];
      {
        float a[32];
        tmem_ld32(tmem + ((uint32_t)(32 * sw_) << 16) + 64u * b, a);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = a[i];
        tmem_ld32(tmem + ((uint32_t)(32 * sw_) << 16) + 64u * b + 32u, a);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[32 + i] = a[i];
      }
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        s[i] = valid ? s[i] * sm_scale : -INFINITY;
        w[i] = s[i];
      }
      float rr[4];
      reduce_scatter16x64<true>(w, lane, rr);
      if (lo_half) {
#pragma unroll
        for (int e = 0; e < 4; ++e) red_m[sw_ * 64 + 4 * hl + e] = rr[e];
      }
      smx_bar();
      if (tid < 64) {
        const float mt = fmaxf(fmaxf(red_m[tid], red_m[64 + tid]), fmaxf(red_m[128 + tid], red_m[192 + tid]));
        m_tile[tid] = mt;
        if (t > 0 && mt > m_run[tid] + kRescaleSlack) atomicOr(&misc[2], 1u);
      }
      smx_bar();
      const bool rescale = t > 0 && (misc[2] & 1u);
      if (tid < 64) {
        const float mt = m_tile[tid];
        if (t == 0) {
          m_run[tid] = mt;
          l_run[tid] = 0.0f;
          fac[tid] = 1.0f;
        } else if (rescale) {
          const float mn = fmaxf(m_run[tid], mt);
          fac[tid] = (m_run[tid] == -INFINITY) ? 0.0f : exp2f((m_run[tid] - mn) * kLog2e);
          m_run[tid] = mn;
          l_run[tid] *= fac[tid];
        }
      }
      smx_bar();
      if (rescale) {
        if (tid == 0) misc[2] = 0;
        // O^T must be complete before it is rescaled: PV of tile t-1
        if (!smx_all(mbar_wait(kempty((t - 1) & 1), ((t - 1) >> 1) & 1))) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) {
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            float o[32];
            const uint32_t ta = tmem + ((uint32_t)(32 * sw_) << 16) + kColO + 64u * mt + 32u * hh;
            tmem_ld32(ta, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= fac[32 * hh + i];
            tmem_st32(ta, o);
          }
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      }
      // probabilities with the running max (<= e^8 between rescales)
      float ps[4];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        s[i] = valid ? exp2f((s[i] - m_run[i]) * kLog2e) : 0.0f;
        w[i] = s[i];
      }
      reduce_scatter16x64<false>(w, lane, ps);
      if (lo_half) {
#pragma unroll
        for (int e = 0; e < 4; ++e) red_l[sw_ * 64 + 4 * hl + e] = ps[e];
      }
      // P^T buffer b is free once PV of tile t-2 is done
      if (t >= 2 && !smx_all(mbar_wait(kempty(b), ((t - 2) >> 1) & 1))) { ok = false; break; }
      if (lo_half) {
        const uint32_t pbase = kOffP + b * kPtBytes + (row >> 3) * 1024u + (row & 7) * 128u;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint4 pk;
          pk.x = pack_bf16x2(s[8 * j + 0], s[8 * j + 1]);
          pk.y = pack_bf16x2(s[8 * j + 2], s[8 * j + 3]);
          pk.z = pack_bf16x2(s[8 * j + 4], s[8 * j + 5]);
          pk.w = pack_bf16x2(s[8 * j + 6], s[8 * j + 7]);
          *reinterpret_cast<uint4*>(sp + pbase + ((j ^ (row & 7)) << 4)) = pk;
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(pfull(b));
      smx_bar();
      if (tid < 64) l_run[tid] += (red_l[tid] + red_l[64 + tid]) + (red_l[128 + tid] + red_l[192 + tid]);
    }
    // epilogue: the last PV completes O^T
    ok = smx_all(ok) && smx_all(mbar_wait(kempty((nt - 1) & 1), ((nt - 1) >> 1) & 1));
    tc_fence_after();
    if (__all_sync(0xffffffffu, ok)) {
      const int chl = 32 * sw_ + lane;                 // channel within a 128-channel tile
#pragma unroll 1
      for (int mt = 0; mt < 4; ++mt) {
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          if (32 * hh >= H) continue;
          float o[32];
          tmem_ld32(tmem + ((uint32_t)(32 * sw_) << 16) + kColO + 64u * mt + 32u * hh, o);
          const int ch = 128 * mt + chl;
          if (nsplit == 1) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int h = 32 * hh + i;
              if (h < H) {
                const float l = l_run[h];
                out[((int64_t)r * H + h) * kD + ch] = f32_to_bf16_rne(l > 0.0f ? o[i] / l : 0.0f);
              }
            }
          } else {
            float* po = part_o + (((int64_t)r * nsplit + split) * H) * kD;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int h = 32 * hh + i;
              if (h < H) po[(int64_t)h * kD + ch] = o[i];
            }
          }
        }
      }
      if (nsplit > 1 && tid < H)
        part_ml[((int64_t)r * nsplit + split) * H + tid] = make_float2(m_run[tid], l_run[tid]);
    }
  }

  // teardown
  const bool all_ok = __syncthreads_and(ok) != 0;
  if (!all_ok) {
    if (tid == 0) raise_error(c.err, CSA2_DEVERR_TIMEOUT);
    // bounded: let the MMAs issued so far drain before TMEM is released
    if (misc[3] != 0) mbar_wait(misc[3], misc[4]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// Merge the S ranges of each (query, head): out = sum_j e^(m_j-M) O_j / sum_j e^(m_j-M) l_j.
// CTA = (query, 4 heads); thread = 8 channels of one head.
__global__ void __launch_bounds__(256) attn_combine_kernel(int H, int nsplit, const float* __restrict__ part_o,
                                                           const float2* __restrict__ part_ml,
                                                           uint16_t* __restrict__ out) {
  const int r = blockIdx.y;
  const int h = blockIdx.x * 4 + (threadIdx.x >> 6);
  const int c8 = (threadIdx.x & 63) * 8;
  if (h >= H) return;
  float M = -INFINITY;
  for (int j = 0; j < nsplit; ++j) {
    const float2 ml = part_ml[((int64_t)r * nsplit + j) * H + h];
    if (ml.y > 0.0f) M = fmaxf(M, ml.x);
  }
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float den = 0.0f;
  if (M != -INFINITY) {
    for (int j = 0; j < nsplit; ++j) {
      const float2 ml = part_ml[((int64_t)r * nsplit + j) * H + h];
      if (!(ml.y > 0.0f)) continue;
      const float wgt = exp2f((ml.x - M) * 1.4426950408889634f);
      den = fmaf(wgt, ml.y, den);
      const float4* src = reinterpret_cast<const float4*>(part_o + (((int64_t)r * nsplit + j) * H + h) * kD + c8);
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

// Ranges per query: enough CTAs to cover the SMs, at most one per 64-row tile.
static int attn_splits(int nq) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int s = nq > 0 ? sms / nq : 1;
  if (s < 1) s = 1;
  if (s > kMaxSplits) s = kMaxSplits;
  return s;
}

size_t attn_workspace_bytes(int nq, int H) {
  const int s = attn_splits(nq);
  if (s == 1) return 0;
  const size_t o = (size_t)nq * s * H * kD * sizeof(float);
  const size_t ml = (size_t)nq * s * H * sizeof(float2);
  return o + ml + 256;
}

cudaError_t attention_set_attributes() {
  return cudaFuncSetAttribute(attn_pipe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kPipeSmem);
}

cudaError_t launch_attention(const CacheView& c, const uint16_t* q, int H, float sm_scale,
                             const int32_t* q_seq, const int32_t* q_vis, const int32_t* idx, int nq,
                             uint16_t* out, void* ws, cudaStream_t st) {
  if (nq == 0) return cudaSuccess;
  if (H % 16 != 0 || H < 16 || H > kHeadsMma) return cudaErrorInvalidValue;
  const int s = attn_splits(nq);
  const int range = (kMaxRows + s - 1) / s;
  float* part_o = reinterpret_cast<float*>(ws);
  float2* part_ml = s > 1 ? reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(ws) +
                                                      (size_t)nq * s * H * kD * sizeof(float))
                          : nullptr;
  attn_pipe_kernel<<<dim3(s, nq), kPipeThreads, kPipeSmem, st>>>(c, q, H, sm_scale, q_seq, q_vis, idx, s,
                                                                 range, out, part_o, part_ml);
  if (s > 1) attn_combine_kernel<<<dim3((H + 3) / 4, nq), 256, 0, st>>>(H, s, part_o, part_ml, out);
  return cudaGetLastError();
}

}  // namespace csa2
