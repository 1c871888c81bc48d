// Seeded synthetic-input generator, device side: the CUDA twin of gen.c.
//
// Same definitions as gen.c (SplitMix64 counter stream, Irwin-Hall(12) normal
// with a single round-to-nearest int->float conversion, RNE to bfloat16), so
// that a workload too large to generate on the host (a 1M-token context) is
// produced on the GPU with the same bits the host generator gives for any row
// the oracle regenerates.  No CSA2 arithmetic lives here.
#include <cstdint>
#include <cuda_runtime.h>

#include "../include/csa2_workload.h"

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ULL;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

__host__ __device__ __forceinline__ uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return mix64(seed ^ mix64(stream + kGamma));
}

__device__ __forceinline__ float normal_at(uint64_t key, uint64_t i) {
  int32_t s = 0;
#pragma unroll
  for (int j = 0; j < 6; ++j) {
    uint64_t h = mix64(key + (6 * i + (uint64_t)j + 1) * kGamma);
    s += (int32_t)(h >> 40) + (int32_t)((h >> 16) & 0xFFFFFFu);
  }
  s -= 6 << 24;
  return __int2float_rn(s) * 0x1p-24f;
}

__device__ __forceinline__ uint16_t to_bf16_rne(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// Batch b uses stream stream0 + b * stream_stride and writes per_batch values
// of that stream, starting at element `start`, to out[b * per_batch + j].
__global__ void fill_normal_bf16_kernel(uint64_t seed, uint64_t stream0, uint64_t stream_stride,
                                        int64_t nbatch, uint64_t per_batch, uint64_t start,
                                        float scale, const float* __restrict__ col_scale,
                                        uint32_t ncols, uint16_t* __restrict__ out) {
  const uint64_t total = (uint64_t)nbatch * per_batch;
  const uint64_t step = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t t = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += step) {
    const uint64_t b = t / per_batch;
    const uint64_t e = start + (t - b * per_batch);
    const uint64_t key = stream_key(seed, stream0 + b * stream_stride);
    float v = normal_at(key, e);
    if (col_scale) v = v * col_scale[e % ncols];
    v = v * scale;
    out[t] = to_bf16_rne(v);
  }
}

}  // namespace

extern "C" int wl_cuda_fill_normal_bf16(uint64_t seed, uint64_t stream0, uint64_t stream_stride,
                                        int64_t nbatch, uint64_t per_batch, uint64_t start,
                                        float scale, const float* col_scale, uint32_t ncols,
                                        uint16_t* out, cudaStream_t stream) {
  if (nbatch < 0 || (nbatch > 0 && per_batch > 0 && out == nullptr)) return 1;
  if (col_scale != nullptr && ncols == 0) return 1;
  const uint64_t total = (uint64_t)nbatch * per_batch;
  if (total == 0) return 0;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  uint64_t blocks = (total + 255) / 256;
  const uint64_t cap = (uint64_t)sms * 16;
  if (blocks > cap) blocks = cap;
  fill_normal_bf16_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
      seed, stream0, stream_stride, nbatch, per_batch, start, scale, col_scale,
      col_scale ? ncols : 1u, out);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
