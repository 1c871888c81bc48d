// Access-pattern ceilings of the B200: kernels that only move the bytes a CSA2
// kernel must move, in the same pattern, so that the benchmark can set each
// CSA2 kernel's time beside the least time that pattern takes on this GPU.
// They compute nothing of the method.  Every loaded 32-bit word is added
// (mod 2^32) into the thread's slot of `sink`, so the sum of all slots equals
// the sum of the words each kernel was asked to read (counted with
// multiplicity): a test checks that against the host.
//
//   csa2c_stream:       a contiguous read (the copy-peak pattern);
//   csa2c_gather_units: random 1-KiB units (the indexer's key units: 8 keys x
//                       128 B), two units per warp in flight, 2 chunks per lane;
//   csa2c_gather_rows:  random 288-B rows (the FP4 cache rows the attention
//                       gathers), 32 rows per warp in flight;
//                       (both number their warps across the CTAs first, so that
//                       a short list still spreads over every SM)
//   csa2c_attn_inputs:  the attention's inputs per CTA: 128 CTAs of 416
//                       threads, CTA b reading query b / 4 (64 KiB) and rows
//                       ids[160 b, 160 b + 160) with the producers' layout
//                       (16 lanes per row), optionally then writing a 64-KiB
//                       slice (the range merge's store);
//   csa2c_cta_load:     n CTAs of 1,024 threads, each reading 64 KiB of
//                       contiguous data (the top-k's load of its scores).
// Bench-side measurement aid, built beside the CSA2 library, not part of it.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint4 ldnc(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t wsum(uint4 v) { return v.x + v.y + v.z + v.w; }

__global__ void __launch_bounds__(256) stream_kernel(const uint4* __restrict__ src, int64_t n16, uint32_t* sink) {
  uint32_t acc = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    const uint4 a = ldnc(src + i), b = ldnc(src + i + stride), c = ldnc(src + i + 2 * stride),
                d = ldnc(src + i + 3 * stride);
    acc += wsum(a) + wsum(b) + wsum(c) + wsum(d);
  }
  for (; i < n16; i += stride) acc += wsum(ldnc(src + i));
  sink[(int64_t)blockIdx.x * blockDim.x + threadIdx.x] = acc;
}

// unit u = ids[u] x 1 KiB; warp w takes units 2w, 2w + 1, then strides by 2 x warps
__global__ void __launch_bounds__(256) gather_units_kernel(const uint4* __restrict__ pool,
                                                           const uint32_t* __restrict__ ids, int n,
                                                           uint32_t* sink) {
  const int lane = threadIdx.x & 31;
  const int gw = (int)((threadIdx.x >> 5) * gridDim.x + blockIdx.x);   // consecutive warps on different CTAs
  const int nw = (int)((gridDim.x * blockDim.x) >> 5);
  uint32_t acc = 0;
  for (int base = 2 * gw; base < n; base += 2 * nw) {
    uint4 v[2][2];
#pragma unroll
    for (int d = 0; d < 2; ++d) {
      if (base + d < n) {
        const uint4* p = pool + (int64_t)ids[base + d] * 64;
        v[d][0] = ldnc(p + lane);
        v[d][1] = ldnc(p + 32 + lane);
      } else {
        v[d][0] = v[d][1] = make_uint4(0, 0, 0, 0);
      }
    }
    acc += wsum(v[0][0]) + wsum(v[0][1]) + wsum(v[1][0]) + wsum(v[1][1]);
  }
  sink[(int64_t)blockIdx.x * blockDim.x + threadIdx.x] = acc;
}

// row u = ids[u] x 288 B (18 chunks); a warp takes 16 rows (288 chunks, 9 per lane)
// per round, two rounds in flight
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ pool,
                                                          const uint32_t* __restrict__ ids, int n,
                                                          uint32_t* sink) {
  const int lane = threadIdx.x & 31;
  const int gw = (int)((threadIdx.x >> 5) * gridDim.x + blockIdx.x);   // consecutive warps on different CTAs
  const int nw = (int)((gridDim.x * blockDim.x) >> 5);
  uint32_t acc = 0;
  for (int base = 32 * gw; base < n; base += 32 * nw) {
    uint4 v[2][9];
#pragma unroll
    for (int d = 0; d < 2; ++d) {
#pragma unroll
      for (int i = 0; i < 9; ++i) {
        const int j = lane + 32 * i;   // chunk j of the round's 16 x 18
        const int u = base + 16 * d + j / 18;
        v[d][i] = u < n ? ldnc(pool + (int64_t)ids[u] * 18 + (j % 18)) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int d = 0; d < 2; ++d)
#pragma unroll
      for (int i = 0; i < 9; ++i) acc += wsum(v[d][i]);
  }
  sink[(int64_t)blockIdx.x * blockDim.x + threadIdx.x] = acc;
}

constexpr int kAttnCtas = 128, kAttnThreads = 416, kRowsPerCta = 160, kQChunks = 4096;

template <bool STORE>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_inputs_kernel(const uint4* __restrict__ q,
                                                                      const uint4* __restrict__ pool,
                                                                      const uint32_t* __restrict__ ids,
                                                                      uint4* __restrict__ part, uint32_t* sink) {
  const int tid = threadIdx.x, b = blockIdx.x;
  uint32_t acc = 0;
  uint4 qv[10];
  const uint4* qs = q + (int64_t)(b >> 2) * kQChunks;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const int e = tid + kAttnThreads * i;
    qv[i] = e < kQChunks ? ldnc(qs + e) : make_uint4(0, 0, 0, 0);
  }
  if (tid < 256) {   // 8 producer warps: 16 half-warps x 10 rows
    const int half = tid >> 4, l16 = tid & 15;
    uint4 rv[10], rt[10];
#pragma unroll
    for (int i = 0; i < 10; ++i) {
      const uint4* rp = pool + (int64_t)ids[kRowsPerCta * b + half * 10 + i] * 18;
      rv[i] = ldnc(rp + l16);
      rt[i] = l16 < 2 ? ldnc(rp + 16 + l16) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 10; ++i) acc += wsum(rv[i]) + wsum(rt[i]);
  }
#pragma unroll
  for (int i = 0; i < 10; ++i) acc += wsum(qv[i]);
  if (STORE) {
    __syncthreads();
    uint4* ps = part + (int64_t)b * kQChunks;
    for (int e = tid; e < kQChunks; e += kAttnThreads) ps[e] = make_uint4(acc, (uint32_t)e, (uint32_t)b, 0u);
  }
  sink[(int64_t)b * kAttnThreads + tid] = acc;
}

__global__ void __launch_bounds__(1024) cta_load_kernel(const uint4* __restrict__ src, uint32_t* sink) {
  const uint4* s = src + (int64_t)blockIdx.x * 4096;
  uint4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = ldnc(s + threadIdx.x + 1024 * i);
  sink[(int64_t)blockIdx.x * 1024 + threadIdx.x] = wsum(v[0]) + wsum(v[1]) + wsum(v[2]) + wsum(v[3]);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

// Sink slots each call writes (the caller's sink must hold at least this many).
long long csa2c_sink_slots(int kernel, int grid) {
  switch (kernel) {
    case 0: case 1: case 2: return (long long)grid * 256;
    case 3: return (long long)kAttnCtas * kAttnThreads;
    default: return (long long)grid * 1024;
  }
}

// 0 on a launch, -1 on a bad argument, else the CUDA error.
int csa2c_stream(const void* src, long long n16, void* sink, int grid, void* stream) {
  if (!src || !sink || n16 < 0 || grid <= 0 || !aligned16(src)) return -1;
  stream_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>((const uint4*)src, n16, (uint32_t*)sink);
  return (int)cudaGetLastError();
}

// ids[i] < (pool bytes) / 1024 for every i < n
int csa2c_gather_units(const void* pool, const void* ids, int n, void* sink, int grid, void* stream) {
  if (!pool || !ids || !sink || n < 0 || grid <= 0 || !aligned16(pool)) return -1;
  gather_units_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>((const uint4*)pool, (const uint32_t*)ids, n,
                                                              (uint32_t*)sink);
  return (int)cudaGetLastError();
}

// ids[i] < (pool bytes) / 288 for every i < n
int csa2c_gather_rows(const void* pool, const void* ids, int n, void* sink, int grid, void* stream) {
  if (!pool || !ids || !sink || n < 0 || grid <= 0 || !aligned16(pool)) return -1;
  gather_rows_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>((const uint4*)pool, (const uint32_t*)ids, n,
                                                             (uint32_t*)sink);
  return (int)cudaGetLastError();
}

// q: 32 x 64 KiB; ids: 128 x 160 row ids (< pool bytes / 288); part (store != 0): 128 x 64 KiB
int csa2c_attn_inputs(const void* q, const void* pool, const void* ids, void* part, void* sink, int store,
                      void* stream) {
  if (!q || !pool || !ids || !sink || (store && !part) || !aligned16(q) || !aligned16(pool) ||
      (store && !aligned16(part)))
    return -1;
  cudaStream_t s = (cudaStream_t)stream;
  if (store)
    attn_inputs_kernel<true><<<kAttnCtas, kAttnThreads, 0, s>>>((const uint4*)q, (const uint4*)pool,
                                                               (const uint32_t*)ids, (uint4*)part, (uint32_t*)sink);
  else
    attn_inputs_kernel<false><<<kAttnCtas, kAttnThreads, 0, s>>>((const uint4*)q, (const uint4*)pool,
                                                                (const uint32_t*)ids, nullptr, (uint32_t*)sink);
  return (int)cudaGetLastError();
}

// src: ncta x 64 KiB
int csa2c_cta_load(const void* src, int ncta, void* sink, void* stream) {
  if (!src || !sink || ncta <= 0 || !aligned16(src)) return -1;
  cta_load_kernel<<<ncta, 1024, 0, (cudaStream_t)stream>>>((const uint4*)src, (uint32_t*)sink);
  return (int)cudaGetLastError();
}

}  // extern "C"
