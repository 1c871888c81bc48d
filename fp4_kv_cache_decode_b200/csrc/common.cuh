// Shared device-side definitions of the CSA2 kernels: cache geometry, paged
// addressing with bounds checks, bf16 helpers and the E4M3/E2M1 decoders.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/csa2.h"

namespace csa2 {

constexpr int kD = CSA2_LATENT_DIM;                   // 512
constexpr int kGroup = CSA2_SCALE_GROUP;              // 16
constexpr int kGroups = kD / kGroup;                  // 32
constexpr int kCodeBytes = kD / 2;                    // 256
constexpr int kRowBytes = CSA2_ROW_BYTES;             // 288
constexpr int kPageTokens = CSA2_PAGE_TOKENS;         // 64
constexpr int kPageBytes = kRowBytes * kPageTokens;   // 18432
constexpr int kIdxHeads = CSA2_IDX_HEADS;             // 4
constexpr int kIdxDim = CSA2_IDX_DIM;                 // 64
constexpr int kIdxRowBytes = kIdxDim * 2;             // 128
constexpr int kIdxPageBytes = kIdxRowBytes * kPageTokens;  // 8192
constexpr int kBlock = CSA2_BLOCK_TOKENS;             // 8
constexpr int kBlocksPerPage = kPageTokens / kBlock;  // 8
constexpr int kBkPageBytes = kBlocksPerPage * kIdxRowBytes;  // 1024
// FP8 indexer keys: 64 E4M3 code bytes per token, the page's 64 fp32 scales after its codes
constexpr int kIdx8RowBytes = kIdxDim;                          // 64
constexpr int kIdx8ScaleOff = kIdx8RowBytes * kPageTokens;      // 4096
constexpr int kIdx8PageBytes = kIdx8ScaleOff + 4 * kPageTokens;  // 4352
constexpr int kPoolBlocks = CSA2_POOL_BLOCKS;         // 2048
constexpr int kTopK = CSA2_TOP_K;                     // 512
constexpr int kWindow = CSA2_WINDOW;                  // 128
constexpr int kReplay = CSA2_REPLAY;                  // 128
constexpr int kMaxRows = kTopK + kWindow;             // 640 attended rows at most

// Kernel-side copy of csa2_cache.
struct CacheView {
  uint8_t* kv;
  uint8_t* idxk;
  uint8_t* bk;
  int64_t n_pages;
  const int32_t* pt;
  int32_t max_pages;
  int32_t batch;
  const int32_t* seq_lens;
  uint32_t* err;
  uint8_t* swa;   // separate sliding-window store [batch][128][288 B], or nullptr
  int idxk_fp8;   // indexer keys: 0 bf16, 1 E4M3 codes + fp32 scale
};

__device__ __forceinline__ void raise_error(uint32_t* err, uint32_t bits) { atomicOr(err, bits); }

#ifdef CSA2_TEST_HOOKS
// Test build only (lib/libcsa2_test.so): while a caller has set this bit of the
// cache's error word, the attention and tensor-core scorer kernels wait on an
// mbarrier that nothing completes, so that a bounded wait runs out and the
// timeout path (error bit, drain, TMEM release) runs on the GPU.
constexpr uint32_t kTestStallBit = 0x80000000u;
__device__ __forceinline__ bool test_stall(const uint32_t* err) {
  return (*reinterpret_cast<const volatile uint32_t*>(err) & kTestStallBit) != 0;
}
#endif

// Page id holding token `tok` of sequence `seq`, or -1 (with an error bit
// raised) when the sequence, the page slot or the page id is out of range.
__device__ __forceinline__ int64_t page_of(const CacheView& c, int seq, int64_t tok) {
  if (seq < 0 || seq >= c.batch) {
    raise_error(c.err, CSA2_DEVERR_SEQ);
    return -1;
  }
  const int64_t slot = tok >> 6;
  if (tok < 0 || slot >= c.max_pages) {
    raise_error(c.err, CSA2_DEVERR_POS);
    return -1;
  }
  const int32_t p = c.pt[(int64_t)seq * c.max_pages + slot];
  if (p < 0 || (int64_t)p >= c.n_pages) {
    raise_error(c.err, CSA2_DEVERR_PAGE);
    return -1;
  }
  return p;
}

__device__ __forceinline__ int seq_len_of(const CacheView& c, int seq) {
  return (seq >= 0 && seq < c.batch) ? c.seq_lens[seq] : 0;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Value of an E4M3 (FN) scale byte with the sign bit clear (codes 0..126).
__device__ __forceinline__ float e4m3_pos_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  if (e == 0) return (float)m * 0x1p-9f;                    // subnormal m/8 * 2^-6
  return __uint_as_float(((e + 120u) << 23) | (m << 20));   // (1 + m/8) * 2^(e-7)
}

// Two E4M3 (FN) bytes, the low byte first, to their exact fp32 values (through
// f16, which holds every E4M3 value).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t pair) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((unsigned short)(pair & 0xFFFFu)));
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// Magnitudes of the E2M1 codes 0..7 (bit 3 is the sign).
__device__ __forceinline__ float e2m1_mag(uint32_t code) {
  // 0, 0.5, 1, 1.5, 2, 3, 4, 6: exponent field e = code>>1, mantissa bit code&1
  const uint32_t e = (code >> 1) & 3u, m = code & 1u;
  if (e == 0) return m ? 0.5f : 0.0f;
  return __uint_as_float(((e + 126u) << 23) | (m << 22));   // (1 + m/2) * 2^(e-1)
}

// Streaming 16-byte global load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Order-preserving map of an fp32 score to uint32 (larger score -> larger
// key); -0 maps like +0 and -inf (the "no candidate" marker) maps to 0.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;
  const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return k <= 0x007FFFFFu ? 0u : k;
}

// Programmatic dependent launch.  Kernels are launched with launch_pdl, so a
// kernel's CTAs may be scheduled while the previous kernel of the stream drains;
// every kernel calls pdl_wait() before it reads anything (an earlier kernel may
// have written it) and then pdl_trigger() so that the next launch can begin.
// Both are no-ops for a launch without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace csa2
