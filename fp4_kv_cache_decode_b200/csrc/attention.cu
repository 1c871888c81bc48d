// CSA2 sparse attention over the FP4 cache on the 5th-generation tensor cores.
//
// A query attends over its selected positions joined with the 128-token
// sliding window (agentnet.co.il, "דיפסיק משיקה את V4.1-פלאש ...", sections
// "CSA2: דחיסה לאורך ציר השכבות" and "ארכיטקטורה שחותכת בחצי את הפריפיל").
// Every query has 640 candidate slots: slot j < 512 holds idx[j] (used when
// 0 <= idx[j] < w0, the window start), slot 512 + i holds position w0 + i
// (used when it is below the visible length v).  The used slots list every
// attended position exactly once.
//
// Work split: the 640 slots of a query are cut into S contiguous ranges, one
// CTA each (S chosen so that the grid fills the GPU; S = 1 for large
// batches); a small batch also splits each query's heads into G groups of
// H / G >= 16, one cluster of S CTAs per (query, group), since heads are
// independent until the output.  A CTA compacts the used slots of its range into a row list and
// walks it in 64-row tiles through a warp-specialised pipeline:
//   * producer warps (8) keep the FP4 bytes of the next two tiles in flight
//     in registers while they decode the current tile to bf16 (16 lanes per
//     288-B row, coalesced) into one of two shared-memory buffers in the UMMA
//     128-byte-swizzle K-major layout; every E2M1 x E4M3 product is exact in
//     bf16 (byte-permute lookup of the E2M1 magnitude, one bf16x2 multiply by
//     the group scale);
//   * one MMA thread issues S^T = K^ . Q^T (tcgen05.mma, M = 64 rows, N = 64
//     heads, K = 512) into one of two TMEM score buffers -- the next tile's
//     QK runs while the current tile's softmax does -- and, once P^T is
//     ready, O^T += V^T . P^T (M = 128 channels x 4, N = 64, K = 64) into a
//     TMEM accumulator that persists across the CTA's tiles (V = K^, read
//     MN-major from the same bytes), plus l += 1^T . P^T (a ones row) so that
//     the softmax denominator comes from the same bf16 weights as O;
//   * softmax warps (4, one per TMEM sub-partition, all 32 lanes busy) keep
//     a running max m per head in base-2 units.  It is moved only when a
//     score exceeds it by more than kSlack2 (then O^T and l are rescaled in
//     place), so the weights 2^(s - m) stay below 2^kSlack2 and the final
//     O / l is exact up to rounding.
// With S = 1 the CTA writes the normalised bf16 output; otherwise every CTA
// of the query's cluster writes its normalised output as an f16 slice to L2
// and its (m, l) per head to the cluster's shared tables, and after one
// cluster barrier each combines 1/S of the channels (log-sum-exp weights).
// Hand-offs use mbarriers (tcgen05.commit for tensor-core completion); every
// wait is bounded and reports CSA2_DEVERR_TIMEOUT instead of hanging.
#include "common.cuh"
#include "tc.cuh"

#include <cuda_fp16.h>

namespace csa2 {

constexpr int kRowTile = 64;                           // attended rows per pipeline step
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
constexpr uint32_t kOnesBytes = 64u * 128u;            // 8 KiB: [64 x 64] bf16, row 0 ones, K-major
constexpr uint32_t kOffQs = 0;
constexpr uint32_t kOffK = kOffQs + kQsBytes;          // two K^ buffers (result staging at the end)
constexpr uint32_t kOffP = kOffK + 2 * kKtBytes;       // two P^T buffers
constexpr uint32_t kOffOnes = kOffP + 2 * kPtBytes;
constexpr uint32_t kOffRedM = kOffOnes + kOnesBytes;   // float [4][64] tile max per warp
constexpr uint32_t kOffRun = kOffRedM + 1024;          // float m_run[64], fac[64], l[64], f[64]
constexpr uint32_t kOffRows = kOffRun + 1024;          // uint32 physical row ids [640]
constexpr uint32_t kOffMl = kOffRows + 4u * kMaxRows;  // float2 [8 ranks][64 heads]: the cluster's (m, l)
constexpr uint32_t kOffBar = kOffMl + 8u * 64u * 8u;   // 9 mbarriers
constexpr uint32_t kOffMisc = kOffBar + 80;            // 44 words: TMEM base, counters
constexpr uint32_t kPipeSmem = kOffBar + 256 + 1024;   // + slack for 1024-B alignment
constexpr uint32_t kTmemCols = 512;                    // S^T 2x64 + O^T 4x64 + l 64 = 448, rounded up
constexpr uint32_t kColO = 128;                        // first O^T column
constexpr uint32_t kColL = 384;                        // l row (TMEM lane 0)
constexpr uint32_t kNoRow = 0xFFFFFFFFu;
constexpr uint32_t kSwaRow = 0x80000000u;              // flag: id = slot of the sliding-window store
constexpr int kRowCacheInts = CSA2_ATTN_ROWS_INTS;      // 640 row ids + 8 range counts per query
static_assert(kRowCacheInts >= kMaxRows + 8, "row cache layout");
constexpr float kSlack2 = 12.0f;                       // base-2 headroom before the max moves

// Optional inputs/outputs of a position-sharded call: a per-query window start
// (the window is [max(v - 128, wstart), v)) and the base-2 log-sum-exp of each
// head's logits over the attended set (-inf when the set is empty).
struct AttnShardIO {
  const int32_t* wstart;
  float* lse2;
};
static_assert(kPipeSmem <= 232448, "shared memory budget");

// Instruction descriptors for tcgen05.mma kind::f16: D fp32 (bits 4-5 = 1),
// A and B f16 (type fields at bits 7-9 and 10-12 = 0), N>>3 at bit 17,
// M>>4 at bit 24; bit 15 / 16 = A / B are MN-major.
constexpr uint32_t kIdescQK = (1u << 4) | ((uint32_t)(kHeadsMma >> 3) << 17) | ((uint32_t)(kRowTile >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 15) | (1u << 16) | ((uint32_t)(kHeadsMma >> 3) << 17) | (8u << 24);
// l: A = ones row (K-major, M = 64), B = P^T (MN-major), N = 64.
constexpr uint32_t kIdescL = (1u << 4) | (1u << 16) | ((uint32_t)(kHeadsMma >> 3) << 17) | ((uint32_t)(64 >> 4) << 24);


#ifdef CSA2_TEST_HOOKS
constexpr uint32_t kPollLimit = 1u << 20;    // test build: the MMA thread gives up sooner
#else
constexpr uint32_t kPollLimit = 1u << 26;    // idle polls of the MMA thread before it gives up
#endif

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

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(d) : "f"(lo), "f"(hi));
  return d;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(d) : "f"(lo), "f"(hi));
  return d;
}

// One code word (8 E2M1 values, channel 2j in the low nibble of byte j) times
// its group scale (f16x2, both halves equal) -> 8 f16 values.  E2M1 -> f16 and
// E4M3 -> f16 are exact hardware conversions, and every product (at most 6
// significant bits, magnitude in [2^-10, 2688]) is exact in f16.
__device__ __forceinline__ uint4 decode8_f16(uint32_t codes, uint32_t scale2) {
  uint32_t d0, d1, d2, d3;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}\n"
      : "=r"(d0), "=r"(d1), "=r"(d2), "=r"(d3)
      : "r"(codes));
  asm("mul.rn.f16x2 %0, %0, %1;" : "+r"(d0) : "r"(scale2));
  asm("mul.rn.f16x2 %0, %0, %1;" : "+r"(d1) : "r"(scale2));
  asm("mul.rn.f16x2 %0, %0, %1;" : "+r"(d2) : "r"(scale2));
  asm("mul.rn.f16x2 %0, %0, %1;" : "+r"(d3) : "r"(scale2));
  return make_uint4(d0, d1, d2, d3);
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

// 32 fp32 TMEM columns from one 16-lane half of a sub-partition (the rows of
// an M = 64 accumulator): thread t < 16 reads lane base + t, columns
// col .. col + 31; thread t >= 16 reads lane base + t - 16, columns
// col + 32 .. col + 63.
__device__ __forceinline__ void tmem_ld16x2(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
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

// 2^x (hardware approximation, relative error ~2^-22; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Max over the 16 lanes of each half-warp, scattered: lane l ends with the
// maxima of elements 2(l%16) and 2(l%16)+1 in v[0], v[1] (30 shuffles).
__device__ __forceinline__ void max_scatter32x16(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < 2 * w; ++i) {
      const float send = up ? v[i] : v[i + 2 * w];
      const float keep = up ? v[i + 2 * w] : v[i];
      v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, w));
    }
  }
}


// Thread-block cluster: barrier over all threads of the cluster, address of
// the same shared-memory offset in CTA `rank`, and accesses through it.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_v2(uint32_t addr, float a, float b) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}


__device__ __forceinline__ uint4 ld_nc16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ld_nc_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// Producer thread layout for one 64-row tile: 16 lanes per row, lane
// `piece` (0..15) takes the 16-B code chunk `piece` (32 channels) and the two
// scale bytes of those channels; thread rsub (0..15) of a piece takes rows
// rsub + 16 it, it = 0..3.  A warp load then covers two rows' 256 contiguous
// code bytes (few cache lines per instruction).
struct RawTile {
  uint4 c[4];       // code chunk of rows rsub + 16 it
  uint32_t s[4];    // the 4-B scale word holding its two scale bytes
};

__device__ __forceinline__ void raw_load(RawTile& R, const uint8_t* __restrict__ kv,
                                         const uint8_t* __restrict__ swa, const uint32_t* rows_s,
                                         int t, int nrow, int rsub, int piece) {
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int li = t * kRowTile + rsub + 16 * it;
    const uint32_t id = li < nrow ? rows_s[li] : kNoRow;
    if (id != kNoRow) {
      const uint8_t* rp = ((id & kSwaRow) ? swa : kv) + (int64_t)(id & ~kSwaRow) * kRowBytes;
      R.c[it] = ld_nc16(rp + piece * 16);
      R.s[it] = ld_nc_u32(rp + kCodeBytes + (piece >> 1) * 4);
    } else {   // zero codes and zero scales decode to zeros
      R.c[it] = make_uint4(0, 0, 0, 0);
      R.s[it] = 0;
    }
  }
}

// Decode into the swizzled K^ buffer at kbuf (channel block kb = piece >> 1,
// 16-B columns 4 (piece & 1) + j).  The four output words are produced in
// the order j = (jj + kb) & 3 so that the 8 lanes of a quarter-warp (same
// row, 4 channel blocks) store to 8 different bank groups.  soff[jj] is the
// byte offset of column 4 (piece & 1) + ((jj + kb) & 3) within the swizzled row.
__device__ __forceinline__ void raw_decode(const RawTile& R, uint8_t* sp, uint32_t kbuf, int rsub, int piece,
                                           const uint32_t (&soff)[4]) {
  const int kb = piece >> 1, rot = kb & 3;
  const uint32_t base = kbuf + (uint32_t)kb * (kRowTile * 128u) + (uint32_t)rsub * 128u;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    // rotate the code words by rot; words 0, 1 use scale byte 0, words 2, 3 byte 1
    uint32_t w0 = R.c[it].x, w1 = R.c[it].y, w2 = R.c[it].z, w3 = R.c[it].w;
    if (rot & 1) { const uint32_t t = w0; w0 = w1; w1 = w2; w2 = w3; w3 = t; }
    if (rot & 2) { uint32_t t = w0; w0 = w2; w2 = t; t = w1; w1 = w3; w3 = t; }
    const uint32_t sc16 = (piece & 1) ? (R.s[it] >> 16) : (R.s[it] & 0xFFFFu);
    uint32_t sc, s0, s1;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(sc) : "h"((unsigned short)sc16));
    s0 = __byte_perm(sc, 0u, 0x1010);
    s1 = __byte_perm(sc, 0u, 0x3232);
    const uint32_t cw[4] = {w0, w1, w2, w3};
    const uint32_t rowb = base + (uint32_t)(16 * it) * 128u;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const uint32_t sj = ((jj + rot) & 2) ? s1 : s0;
      *reinterpret_cast<uint4*>(sp + rowb + soff[jj]) = decode8_f16(cw[jj], sj);
    }
  }
}

// Rank `split` of a query's cluster combines channels [split C, (split + 1) C),
// C = 512 / S, of the S normalised f16 slices [S][H][512] in `part`: slice j
// enters with weight 2^(m_j - M) l_j / L (M the largest m_j of the ranks that
// attended something, L the sum of 2^(m_j - M) l_j), read from the cluster's
// (m, l) table `ml` [S][64].  Output bf16.  Task = (head, 8 channels); a
// thread's tasks are tid + 416 t, and all of their loads (at most 16 x 16 B)
// are in flight before the weights are formed.
template <int S>
__device__ __forceinline__ void reduce_slices(const uint16_t* __restrict__ part, uint16_t* __restrict__ out,
                                              const float2* ml, int r, int split, int H, int tid) {
  constexpr int nch = kD / S, c8n = nch / 8;
  constexpr int kTasks = (kHeadsMma * c8n + kPipeThreads - 1) / kPipeThreads;   // per thread at H = 64
  const int ntask = H * c8n;
  uint4 xs[kTasks][S];
#pragma unroll
  for (int t = 0; t < kTasks; ++t) {
    const int task = tid + t * kPipeThreads;
    if (task < ntask) {
      const int h = task / c8n, ch0 = split * nch + 8 * (task % c8n);
#pragma unroll
      for (int j = 0; j < S; ++j)   // L2 only: written by this grid
        xs[t][j] = __ldcg(reinterpret_cast<const uint4*>(part + (((int64_t)r * S + j) * H + h) * kD + ch0));
    }
  }
#pragma unroll
  for (int t = 0; t < kTasks; ++t) {
    const int task = tid + t * kPipeThreads;
    if (task < ntask) {
      const int h = task / c8n, ch0 = split * nch + 8 * (task % c8n);
      float wj[S], M = -INFINITY, L = 0.0f;
#pragma unroll
      for (int j = 0; j < S; ++j) {
        const float2 x = ml[j * 64 + h];
        if (x.y > 0.0f) M = fmaxf(M, x.x);
      }
#pragma unroll
      for (int j = 0; j < S; ++j) {
        const float2 x = ml[j * 64 + h];
        wj[j] = x.y > 0.0f ? ex2(x.x - M) * x.y : 0.0f;
        L += wj[j];
      }
      const float inv = L > 0.0f ? 1.0f / L : 0.0f;
      float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int j = 0; j < S; ++j) {
        const float g = wj[j] * inv;
        const uint32_t w[4] = {xs[t][j].x, xs[t][j].y, xs[t][j].z, xs[t][j].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
          acc[2 * k] = fmaf(g, f2.x, acc[2 * k]);
          acc[2 * k + 1] = fmaf(g, f2.y, acc[2 * k + 1]);
        }
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      *reinterpret_cast<uint4*>(out + ((int64_t)r * H + h) * kD + ch0) = o;
    }
  }
}

__global__ void __launch_bounds__(kPipeThreads, 1)
attn_pipe_kernel(CacheView c, const uint16_t* __restrict__ q, int H, float sm_scale,
                 const int32_t* __restrict__ q_seq, const int32_t* __restrict__ q_vis,
                 const int32_t* __restrict__ idx, int nsplit, int range_slots, int groups,
                 uint16_t* __restrict__ out, uint16_t* __restrict__ part, int32_t* __restrict__ rcache, int rmode,
                 AttnShardIO shard) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw_s = (uint32_t)__cvta_generic_to_shared(smem_raw);
  const uint32_t sb = (raw_s + 1023u) & ~1023u;            // 1024-B aligned base (swizzle atoms)
  uint8_t* const sp = smem_raw + (sb - raw_s);
  float* const red_m = reinterpret_cast<float*>(sp + kOffRedM);
  float* const m_run = reinterpret_cast<float*>(sp + kOffRun);   // base-2 running max per head
  float* const fac = m_run + 64;
  float* const l_s = m_run + 128;
  float* const f_s = m_run + 192;                                 // output factor per head
  float2* const lse_ml = reinterpret_cast<float2*>(sp + kOffRedM);  // epilogue: final (M, L) per head
  uint32_t* const rows_s = reinterpret_cast<uint32_t*>(sp + kOffRows);
  // [0] TMEM base, [1] last barrier the MMA thread committed to (0: none), [2] its parity,
  // [4 + w] used-slot count of warp w, [20 + w] largest |q| bits seen by warp w
  uint32_t* const misc = reinterpret_cast<uint32_t*>(sp + kOffMisc);
  const uint32_t bar0 = sb + kOffBar;
  auto kfull = [&](int b) { return bar0 + 8u * b; };
  auto kempty = [&](int b) { return bar0 + 16u + 8u * b; };
  auto sfull = [&](int b) { return bar0 + 32u + 8u * b; };
  auto pfull = [&](int b) { return bar0 + 48u + 8u * b; };
  const uint32_t qready = bar0 + 64u;

  const int split = blockIdx.x;                            // rank in the query's cluster
  // head group g of query r: heads [g H, (g + 1) H) of its groups x H.  The
  // query, output and log-sum-exp rows of (r, g) are row rv of those arrays
  // viewed as [nq x groups][H]; the positions, index set and row cache are r's.
  const int rv = blockIdx.y;
  const int r = rv / groups;
  const bool rows_owner = rv - r * groups == 0;            // records the resolved rows
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t* idx_row = idx + (int64_t)r * kTopK;
  // the cluster's CTAs all run before any touches another's shared memory:
  // arrive now, wait just before the first remote access
  if (nsplit > 1) cluster_arrive_relaxed();

  // the query's bf16 rows, 16-B chunk e = tid + kPipeThreads * i (heads >= H read as zero);
  // they are scaled by 2^qexp and stored as f16 once the largest magnitude is known
  constexpr int kQChunks = kHeadsMma * (kD / 8);                     // 4096
  constexpr int kQPerThread = (kQChunks + kPipeThreads - 1) / kPipeThreads;   // 10
  uint4 qv[kQPerThread];
  {
    const uint4* qsrc = reinterpret_cast<const uint4*>(q + (int64_t)rv * H * kD);
#pragma unroll
    for (int i = 0; i < kQPerThread; ++i) {
      const int e = tid + kPipeThreads * i;
      qv[i] = (e < kQChunks && (e >> 6) < H) ? ld_nc16(qsrc + e) : make_uint4(0, 0, 0, 0);
    }
  }
  // ones row for the softmax denominator: row 0 of a K-major [64 x 64] f16 tile,
  // fenced for the tensor core
  for (int e = tid; e < (int)(kOnesBytes / 16); e += kPipeThreads)
    *reinterpret_cast<uint4*>(sp + kOffOnes + 16 * e) =
        e < 8 ? make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u) : make_uint4(0, 0, 0, 0);
  fence_async_smem();

  // this CTA's candidate slots; thread tid takes slots lo + 2 tid and lo + 2 tid + 1
  const int lo = split * range_slots;
  const int hi = min(lo + range_slots, kMaxRows);
  const int s0 = lo + 2 * tid;
  // row cache of this query: ids of range j at [j * range_slots ...), counts at [640 + j]
  int32_t* const rc_row = rcache ? rcache + (int64_t)r * kRowCacheInts : nullptr;
  bool u0 = false, u1 = false;   // slot used
  uint32_t id0 = kNoRow, id1 = kNoRow;
  if (rmode == 2) {   // the rows a Full / Reindex call resolved for this set and range
    // the ids load together with the count (slots past it hold stale ids, dropped below)
    const int32_t c0 = s0 < hi ? rc_row[s0] : -1, c1 = s0 + 1 < hi ? rc_row[s0 + 1] : -1;
    const int nrow_c = rc_row[kMaxRows + split];
    u0 = s0 < hi && s0 - lo < nrow_c;
    u1 = s0 + 1 < hi && s0 + 1 - lo < nrow_c;
    if (u0) id0 = (uint32_t)c0;
    if (u1) id1 = (uint32_t)c1;
  } else {
    int32_t e0 = -1, e1 = -1;
    if (s0 < hi && s0 < kTopK) e0 = idx_row[s0];
    if (s0 + 1 < hi && s0 + 1 < kTopK) e1 = idx_row[s0 + 1];
    const int seq = q_seq[r];
    const int64_t v = q_vis ? (int64_t)q_vis[r] : (int64_t)seq_len_of(c, seq);
    // window [w0, v): the last 128 visible positions, or from a given start
    // (at most 128 positions; a start at v leaves the window empty)
    int64_t w0 = v > kWindow ? v - kWindow : 0;
    if (shard.wstart) w0 = max(w0, min(v, (int64_t)max(0, shard.wstart[r])));
    auto slot_pos = [&](int sl, int32_t e) -> int64_t {   // attended position of a slot, -1 if unused
      if (sl >= hi) return -1;
      if (sl < kTopK) {
        if (e >= v) raise_error(c.err, CSA2_DEVERR_POS);
        return (e >= 0 && e < w0) ? (int64_t)e : -1;
      }
      const int64_t p = w0 + (sl - kTopK);
      return p < v ? p : -1;
    };
    const int64_t p0 = slot_pos(s0, e0), p1 = slot_pos(s0 + 1, e1);
    u0 = p0 >= 0;
    u1 = p1 >= 0;
    // physical row: a sequence's last 128 entries come from the sliding-window
    // store when there is one, every other entry from its cache page
    const int64_t swa_from = c.swa ? (int64_t)seq_len_of(c, seq) - kReplay : INT64_MAX;
    auto row_id = [&](int64_t p) -> uint32_t {
      if (p >= swa_from) return kSwaRow | (uint32_t)(seq * kReplay + (int)(p & (kReplay - 1)));
      const int64_t pg = page_of(c, seq, p);
      return pg >= 0 ? (uint32_t)(pg * kPageTokens + (p & (kPageTokens - 1))) : kNoRow;
    };
    if (u0) id0 = row_id(p0);
    if (u1) id1 = row_id(p1);
  }
  // largest |q| of the warp (the loads above were in flight meanwhile)
  uint32_t qmax = 0;   // as bf16 bits: magnitudes order like their bit patterns
  {
#pragma unroll
    for (int i = 0; i < kQPerThread; ++i) {
      qmax = __vmaxu2(qmax, qv[i].x & 0x7FFF7FFFu);
      qmax = __vmaxu2(qmax, qv[i].y & 0x7FFF7FFFu);
      qmax = __vmaxu2(qmax, qv[i].z & 0x7FFF7FFFu);
      qmax = __vmaxu2(qmax, qv[i].w & 0x7FFF7FFFu);
    }
    qmax = max(qmax & 0xFFFFu, qmax >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qmax = max(qmax, __shfl_xor_sync(0xffffffffu, qmax, o));
  }
  // compact the used slots (in slot order) into rows_s
  const uint32_t cnt = (u0 ? 1u : 0u) + (u1 ? 1u : 0u);
  uint32_t incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) misc[4 + warp] = incl;
  if (lane == 0) misc[20 + warp] = qmax;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sb + kOffMisc),
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
    mbar_init(qready, kPipeThreads);
#ifdef CSA2_TEST_HOOKS
    mbar_init(bar0 + 72u, 1);   // completed by nothing: the test stall waits on it
#endif
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    misc[1] = 0;
    misc[2] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  uint32_t before = 0, total = 0;
#pragma unroll 1
  for (int w = 0; w <= kMmaWarp; ++w) {
    const uint32_t x = misc[4 + w];
    before += w < warp ? x : 0u;
    total += x;
    qmax = max(qmax, misc[20 + w]);
  }
  {
    const uint32_t at = before + incl - cnt;
    if (u0) rows_s[at] = id0;
    if (u1) rows_s[at + (u0 ? 1u : 0u)] = id1;
    if (rmode == 1 && rows_owner) {   // record them for the Reuse layers
      if (u0) rc_row[lo + at] = (int32_t)id0;
      if (u1) rc_row[lo + at + (u0 ? 1u : 0u)] = (int32_t)id1;
      if (tid == 0) rc_row[kMaxRows + split] = (int32_t)total;
    }
  }
  // Q in f16 scaled by 2^qexp so that the largest |q| lies in [2^14, 2^15):
  // exact for every element of magnitude >= 2^-28 of the largest; the scores
  // are scaled back in the softmax.
  const int qexp = qmax == 0 ? 0 : max(-100, min(100, 141 - (int)(qmax >> 7)));
  auto store_q = [&]() {   // this thread's Q chunks -> f16, swizzled K-major; then signal
    const float qs = __uint_as_float((uint32_t)(127 + qexp) << 23);
#pragma unroll
    for (int i = 0; i < kQPerThread; ++i) {
      const int e = tid + kPipeThreads * i;
      if (e < kQChunks) {
        const int h = e >> 6, c16 = e & 63, kb = c16 >> 3, j = c16 & 7;
        const uint32_t off = kOffQs + kb * (kHeadsMma * 128u) + (h >> 3) * 1024u + (h & 7) * 128u +
                             ((j ^ (h & 7)) << 4);
        uint4 o;
        o.x = pack_f16x2(bf16_lo(qv[i].x) * qs, bf16_hi(qv[i].x) * qs);
        o.y = pack_f16x2(bf16_lo(qv[i].y) * qs, bf16_hi(qv[i].y) * qs);
        o.z = pack_f16x2(bf16_lo(qv[i].z) * qs, bf16_hi(qv[i].z) * qs);
        o.w = pack_f16x2(bf16_lo(qv[i].w) * qs, bf16_hi(qv[i].w) * qs);
        *reinterpret_cast<uint4*>(sp + off) = o;
      }
    }
    fence_async_smem();
    mbar_arrive(qready);
  };
  const int nrow = (int)total;
  const int nt = (nrow + kRowTile - 1) / kRowTile;
  const uint32_t tmem = misc[0];
  __syncthreads();   // rows_s complete
  bool ok = true;

  if (warp >= kSoftmaxWarps && warp < kMmaWarp) {
    // ---------------- producers: gather + decode ----------------
    const int ptid = tid - kSmxThreads;
    const int piece = ptid & 15, rsub = ptid >> 4;
    uint32_t soff[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
      soff[jj] = (uint32_t)((((piece & 1) * 4 + ((jj + (piece >> 1)) & 3)) ^ (rsub & 7)) << 4);
    // tile t's bytes sit in A (t even) or B (t odd); once tile t is decoded its
    // registers take tile t + 2, about one pipeline step ahead of its decode
    // (two buffers keep the loop body small: three would triple the code)
    RawTile A, B;
    if (nt > 0) raw_load(A, c.kv, c.swa, rows_s, 0, nrow, rsub, piece);
    if (nt > 1) raw_load(B, c.kv, c.swa, rows_s, 1, nrow, rsub, piece);
    store_q();
    auto step = [&](int t, RawTile& D) -> bool {
      const int b = t & 1;
      if (t >= 2 && !mbar_wait(kempty(b), ((t - 2) >> 1) & 1)) return false;
      raw_decode(D, sp, kOffK + b * kKtBytes, rsub, piece, soff);
      fence_async_smem();
      mbar_arrive(kfull(b));
      if (t + 2 < nt) raw_load(D, c.kv, c.swa, rows_s, t + 2, nrow, rsub, piece);
      return true;
    };
#pragma unroll 1
    for (int t = 0; t < nt; t += 2) {
      if (!(ok = step(t, A)) || t + 1 >= nt) break;
      if (!(ok = step(t + 1, B))) break;
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issue (one thread) ----------------
    // QK(t) and PV(t) are issued as soon as their inputs are ready, in
    // whichever order they become ready: QK(t) needs tile t decoded and the
    // S buffer free (PV(t-2) issued); PV(t) needs P(t).
    store_q();
    if (lane == 0) {
      ok = mbar_wait(qready, 0);
#ifdef CSA2_TEST_HOOKS
      const bool stall = test_stall(c.err);
#endif
      int nqk = 0, npv = 0;
      uint32_t idle = 0;
      while (ok && npv < nt) {
        bool progressed = false;
        if (npv < nqk && mbar_test(pfull(npv & 1), (npv >> 1) & 1)) {
          const int t = npv, b = t & 1;
          tc_fence_after();
          // descriptors advance by plain adds of (byte offset >> 4) to the start field
          const uint64_t a0 = smem_desc(sb + kOffK + b * kKtBytes, kRowTile * 128u, 1024u);
          const uint64_t p0 = smem_desc(sb + kOffP + b * kPtBytes, 8192u, 1024u);
          const uint64_t o0 = smem_desc(sb + kOffOnes, 16u, 1024u);
          const uint32_t acc = t > 0 ? 1u : 0u;
#pragma unroll
          for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_f16(tmem + kColO + 64u * mt, a0 + (((2 * mt) * (kRowTile * 128u) + ks * 2048u) >> 4),
                      p0 + ((ks * 2048u) >> 4), kIdescPV, (acc | ks) ? 1u : 0u);
          }
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16(tmem + kColL, o0 + ((ks * 32u) >> 4), p0 + ((ks * 2048u) >> 4), kIdescL, (acc | ks) ? 1u : 0u);
          mma_commit(kempty(b));
          misc[1] = kempty(b);
          misc[2] = (t >> 1) & 1;
          ++npv;
          progressed = true;
        }
        if (nqk < nt && nqk <= npv + 1 && mbar_test(kfull(nqk & 1), (nqk >> 1) & 1)) {
          const int t = nqk, b = t & 1;
          tc_fence_after();
          const uint64_t a0 = smem_desc(sb + kOffK + b * kKtBytes, 16u, 1024u);
          const uint64_t q0 = smem_desc(sb + kOffQs, 16u, 1024u);
#pragma unroll
          for (int kb = 0; kb < 8; ++kb) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_f16(tmem + 64u * b, a0 + ((kb * (kRowTile * 128u) + ks * 32u) >> 4),
                      q0 + ((kb * (kHeadsMma * 128u) + ks * 32u) >> 4), kIdescQK, (kb | ks) ? 1u : 0u);
          }
          mma_commit(sfull(b));
          misc[1] = sfull(b);
          misc[2] = (t >> 1) & 1;
          ++nqk;
          progressed = true;
#ifdef CSA2_TEST_HOOKS
          // test stall after the first QK: a wait that runs out with an MMA committed
          if (stall && nqk == 1 && !test_stall_wait(bar0 + 72u)) ok = false;
#endif
        }
        if (progressed) idle = 0;
        else if (++idle > kPollLimit) ok = false;
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax warps 0..3 ----------------
    store_q();
    const int w = warp;                                // TMEM sub-partition == warp
    const int rl = lane & 15, hh = lane >> 4;          // tile row 16 w + rl, heads 32 hh .. 32 hh + 31
    const int row = 16 * w + rl;
    constexpr float kLog2e = 1.4426950408889634f;
    const float scale2 = sm_scale * kLog2e * __uint_as_float((uint32_t)(127 - qexp) << 23);
    const float* mr = m_run + 32 * hh;
    const uint32_t lane_base = (uint32_t)(32 * w) << 16;
    for (int t = 0; t < nt && ok; ++t) {
      const int b = t & 1;
      if (!smx_all(mbar_wait(sfull(b), (t >> 1) & 1))) { ok = false; break; }
      tc_fence_after();
      float s[32];
      tmem_ld16x2(tmem + lane_base + 64u * b, s);
      const bool valid = t * kRowTile + row < nrow;
#pragma unroll
      for (int i = 0; i < 32; ++i) s[i] = valid ? s[i] * scale2 : -INFINITY;
      bool slow = t == 0;
      if (!slow) {
        bool exceed = false;
#pragma unroll
        for (int i = 0; i < 32; ++i) exceed |= s[i] > mr[i] + kSlack2;
        slow = !smx_all(!exceed);
      }
      if (slow) {   // move the running max (uniform over the softmax warps)
        float x[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = s[i];
        max_scatter32x16(x, lane);
        red_m[w * 64 + 32 * hh + 2 * rl] = x[0];
        red_m[w * 64 + 32 * hh + 2 * rl + 1] = x[1];
        smx_bar();
        if (tid < 64) {
          const float mt = fmaxf(fmaxf(red_m[tid], red_m[64 + tid]), fmaxf(red_m[128 + tid], red_m[192 + tid]));
          if (t == 0) {
            m_run[tid] = mt;
            fac[tid] = 1.0f;
          } else {
            const float mn = fmaxf(m_run[tid], mt);
            fac[tid] = ex2(m_run[tid] - mn);
            m_run[tid] = mn;
          }
        }
        smx_bar();
        if (t > 0) {
          // O^T and l must be complete before they are rescaled: PV of tile t-1
          if (!smx_all(mbar_wait(kempty((t - 1) & 1), ((t - 1) >> 1) & 1))) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int ct = 0; ct < 5; ++ct) {
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
              float o[32];
              const uint32_t ta = tmem + lane_base + (ct < 4 ? kColO + 64u * ct : kColL) + 32u * h2;
              tmem_ld32(ta, o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] *= fac[32 * h2 + i];
              tmem_st32(ta, o);
            }
          }
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        }
      }
      // weights 2^(s - m) <= 2^kSlack2 (0 for unused rows)
#pragma unroll
      for (int i = 0; i < 32; ++i) s[i] = ex2(s[i] - mr[i]);
      // P^T buffer b is free once PV of tile t-2 is done
      if (t >= 2 && !smx_all(mbar_wait(kempty(b), ((t - 2) >> 1) & 1))) { ok = false; break; }
      {
        const uint32_t pbase = kOffP + b * kPtBytes + (row >> 3) * 1024u + (row & 7) * 128u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 pk;
          pk.x = pack_f16x2(s[8 * j + 0], s[8 * j + 1]);
          pk.y = pack_f16x2(s[8 * j + 2], s[8 * j + 3]);
          pk.z = pack_f16x2(s[8 * j + 4], s[8 * j + 5]);
          pk.w = pack_f16x2(s[8 * j + 6], s[8 * j + 7]);
          *reinterpret_cast<uint4*>(sp + pbase + (((4 * hh + j) ^ (row & 7)) << 4)) = pk;
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(pfull(b));
    }
    // epilogue: the last PV completes O^T and l
    ok = smx_all(ok) && (nt == 0 || smx_all(mbar_wait(kempty((nt - 1) & 1), ((nt - 1) >> 1) & 1)));
    tc_fence_after();
    if (ok) {
      if (nt > 0) {
        if (w == 0) {   // l sits in TMEM lane 0
          float a[32];
          tmem_ld32(tmem + kColL, a);
          if (lane == 0) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(l_s + i) = make_float4(a[i], a[i + 1], a[i + 2], a[i + 3]);
          }
          tmem_ld32(tmem + kColL + 32u, a);
          if (lane == 0) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(l_s + 32 + i) = make_float4(a[i], a[i + 1], a[i + 2], a[i + 3]);
          }
        }
      } else if (tid < 64) {   // nothing attended in this range
        l_s[tid] = 0.0f;
        m_run[tid] = -INFINITY;
      }
    }
  }

  const bool all_ok = __syncthreads_and(ok) != 0;
  if (!all_ok) {
    if (tid == 0) raise_error(c.err, CSA2_DEVERR_TIMEOUT);
    // bounded: let the MMAs issued so far drain before TMEM is read or released
    if (misc[1] != 0) mbar_wait(misc[1], misc[2]);
  }

  // ---- output ----
  // Every rank writes its normalised O / l: bf16 to `out` with one range per
  // query (nsplit == 1), else f16 to its slice of `part` (shared memory is too
  // slow a path between SMs for 100+ KiB) while its (m, l) per head goes to
  // every rank's table; one cluster barrier later rank j combines channels
  // [j C, (j + 1) C), C = 512 / nsplit, of the nsplit slices by their
  // log-sum-exp weights.  f16 keeps each slice to 2^-11 relative, below the
  // final bf16 rounding.
  if (nsplit > 1) {
    cluster_wait();   // every rank of the cluster runs
    if (tid < 64) {   // (m, l) of this rank per head (l = 0: nothing to add)
      const float mj = all_ok ? m_run[tid] : -INFINITY, lj = all_ok ? l_s[tid] : 0.0f;
      const uint32_t slot = sb + kOffMl + 8u * (uint32_t)(split * 64 + tid);
      for (int j = 0; j < nsplit; ++j) st_cluster_v2(map_shared(slot, (uint32_t)j), mj, lj);
    }
  }
  if (tid < 64) {
    const bool have = all_ok && l_s[tid] > 0.0f;
    f_s[tid] = have ? 1.0f / l_s[tid] : 0.0f;
    lse_ml[tid] = make_float2(have ? m_run[tid] : -INFINITY, have ? l_s[tid] : 0.0f);
  }
  __syncthreads();
  // the idle MMA warp writes the log-sum-exp of a sharded call with one range per query
  if (warp == kMmaWarp && shard.lse2 != nullptr && nsplit == 1) {
    for (int h = lane; h < H; h += 32) {
      const float2 ml = lse_ml[h];
      shard.lse2[(int64_t)rv * H + h] = ml.y > 0.0f ? ml.x + __log2f(ml.y) : -INFINITY;
    }
  }
  // f . O^T straight from TMEM to global [H][512]: the lanes of a warp hold 32
  // consecutive channels, so each 2-B store instruction writes one 64-B run.
  // Warps 0..11 share the work, three per TMEM sub-partition (warp % 4).
  tc_fence_after();   // the last PV's completion was observed before the barriers above
  if (warp < kMmaWarp) {
    uint16_t* dst = nsplit == 1 ? out + (int64_t)rv * H * kD : part + ((int64_t)rv * nsplit + split) * H * kD;
    const int sub = warp & 3;
#pragma unroll 1
    for (int pr = warp >> 2; pr < 8; pr += 3) {   // (channel tile mt, head half h2)
      const int mt = pr >> 1, h2 = pr & 1;
      if (32 * h2 >= H) continue;
      const int ch = 128 * mt + 32 * sub + lane;
      float o[32];
      if (all_ok && nt > 0) {
        tmem_ld32(tmem + ((uint32_t)(32 * sub) << 16) + kColO + 64u * mt + 32u * h2, o);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.0f;
      }
      float fv[32];   // factors in registers: the stores below may not delay their loads
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4*>(&fv[i]) = *reinterpret_cast<const float4*>(f_s + 32 * h2 + i);
#pragma unroll
      for (int i = 0; i < 32; i += 2) {   // two heads per packed conversion
        const uint32_t pk = nsplit == 1 ? pack_bf16x2(o[i] * fv[i], o[i + 1] * fv[i + 1])
                                        : pack_f16x2(o[i] * fv[i], o[i + 1] * fv[i + 1]);
        const int h = 32 * h2 + i;
        if (h < H) dst[h * kD + ch] = (uint16_t)(pk & 0xFFFFu);
        if (h + 1 < H) dst[(h + 1) * kD + ch] = (uint16_t)(pk >> 16);
      }
    }
  }
  if (nsplit > 1) {
    cluster_sync_all();   // every rank's slice is in global memory and its (m, l) in every table
    const float2* ml = reinterpret_cast<const float2*>(sp + kOffMl);
    if (shard.lse2 != nullptr && split == 0 && tid < H) {   // log-sum-exp over the cluster
      float M = -INFINITY, L = 0.0f;
      for (int j = 0; j < nsplit; ++j)
        if (ml[j * 64 + tid].y > 0.0f) M = fmaxf(M, ml[j * 64 + tid].x);
      for (int j = 0; j < nsplit; ++j) {
        const float2 x = ml[j * 64 + tid];
        if (x.y > 0.0f) L += ex2(x.x - M) * x.y;
      }
      shard.lse2[(int64_t)rv * H + tid] = L > 0.0f ? M + __log2f(L) : -INFINITY;
    }
    if (nsplit == 2) reduce_slices<2>(part, out, ml, rv, split, H, tid);
    else if (nsplit == 4) reduce_slices<4>(part, out, ml, rv, split, H, tid);
    else reduce_slices<8>(part, out, ml, rv, split, H, tid);
  }

  // teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

}  // namespace csa2

// ---- launchers used by api.cu ----
namespace csa2 {

// Cluster sizes that fit one query per cluster in a single wave, per device.
static int g_max_clusters[8][4];   // [device][log2 cluster size] (entries 1..3 used)

// Largest range count any launch may use for nq queries: a power of two
// <= 8 with ranges x nq <= 148 (the SM count the workspace is sized for).
static int attn_split_bound(int nq) {
  int s = 8;
  while (s > 1 && (int64_t)s * nq > 148) s >>= 1;
  return s;
}

// Co-resident clusters of s CTAs (s = 1: one CTA per SM).
static int attn_cluster_cap(int dev, int s) {
  if (s == 1) {
    int sms = 0;
    return cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? sms : 0;
  }
  return g_max_clusters[dev][s == 8 ? 3 : s == 4 ? 2 : 1];
}

// Head groups per query for s ranges: the largest divisor G of H / 16 for
// which nq x G clusters of s still fit at once (a query's heads are
// independent until the output; 16 heads is the least the P.V product's N
// takes).
static int attn_head_groups(int dev, int nq, int H, int s) {
  const int cap = attn_cluster_cap(dev, s);
  int best = 1;
  for (int g = 2; g <= H / 16; ++g)
    if ((H / 16) % g == 0 && (int64_t)nq * g <= cap) best = g;
  return best;
}

// Ranges per query: the largest cluster size whose clusters all fit at once
// (fewer rows per CTA shorten its pipeline; head groups then fill the SMs
// left idle -- trading ranges for groups, e.g. 2 ranges x 4 groups instead of
// 4 x 1 at 17 queries, measured slower: 20.2 against 18.8 us per launch).
static int attn_splits(int nq) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 8) return 1;
  const int bound = attn_split_bound(nq);
  for (int lg = 3; lg >= 1; --lg)
    if ((1 << lg) <= bound && nq <= g_max_clusters[dev][lg]) return 1 << lg;
  return 1;
}

size_t attn_workspace_bytes(int nq, int H) {
  const int s = attn_split_bound(nq);
  return s > 1 ? (size_t)nq * s * H * kD * sizeof(uint16_t) + 256 : 0;
}

cudaError_t attention_set_attributes() {
  cudaError_t e = cudaFuncSetAttribute(attn_pipe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kPipeSmem);
  if (e != cudaSuccess) return e;
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev < 0 || dev >= 8) return cudaSuccess;
  for (int lg = 1; lg <= 3; ++lg) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1 << lg, 1);
    cfg.blockDim = dim3(kPipeThreads);
    cfg.dynamicSmemBytes = kPipeSmem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1u << lg;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, attn_pipe_kernel, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    g_max_clusters[dev][lg] = n;
  }
  return cudaSuccess;
}

int attn_splits_for(int nq) { return attn_splits(nq); }

cudaError_t launch_attention(const CacheView& c, const uint16_t* q, int H, float sm_scale,
                             const int32_t* q_seq, const int32_t* q_vis, const int32_t* idx, int nq,
                             uint16_t* out, void* ws, int32_t* rcache, int rmode, int s, cudaStream_t st,
                             const int32_t* wstart, float* lse2) {
  if (nq == 0) return cudaSuccess;
  if (H % 16 != 0 || H < 16 || H > kHeadsMma) return cudaErrorInvalidValue;
  if (s != 1 && s != 2 && s != 4 && s != 8) return cudaErrorInvalidValue;
  if (!rcache) rmode = 0;
  const int range = (kMaxRows + s - 1) / s;
  int dev = 0;
  const int groups = cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 8 ? attn_head_groups(dev, nq, H, s) : 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(s, nq * groups);
  cfg.blockDim = dim3(kPipeThreads);
  cfg.dynamicSmemBytes = kPipeSmem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see launch_pdl
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = (unsigned)s;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = s > 1 ? 2 : 1;
  const AttnShardIO shard{wstart, lse2};
  return cudaLaunchKernelEx(&cfg, attn_pipe_kernel, c, q, H / groups, sm_scale, q_seq, q_vis, idx, s, range,
                            groups, out, reinterpret_cast<uint16_t*>(ws), rcache, rmode, shard);
}

}  // namespace csa2
