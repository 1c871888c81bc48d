/*
 * csa2_workload.h -- seeded synthetic inputs for the CSA2 workloads.
 *
 * Not part of the CSA2 method: this is the input generator that the parity
 * tests, the benchmark and the CPU oracle share.  Two libraries implement it
 * with identical bits: libcsa2_workload_host.so (workload/gen.c) and
 * libcsa2_workload_cuda.so (workload/gen_device.cu).
 *
 * Stream definition (both sides):
 *   key(seed, s)   = mix64(seed ^ mix64(s + 0x9E3779B97F4A7C15))
 *   u64(key, i)    = mix64(key + (i + 1) * 0x9E3779B97F4A7C15)     (mod 2^64)
 *   normal(key, i) = (S - 6*2^24) * 2^-24 with S the sum of the twelve 24-bit
 *                    fields (bits 40..63, 16..39) of u64(key, 6i+j), j=0..5;
 *                    one RNE int->float conversion
 *   mix64          = the SplitMix64 output finaliser (Steele/Lea/Flood 2014)
 */
#ifndef CSA2_WORKLOAD_H
#define CSA2_WORKLOAD_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- host library (libcsa2_workload_host.so) ---- */
uint64_t wl_key(uint64_t seed, uint64_t stream);
uint64_t wl_u64(uint64_t key, uint64_t i);
uint64_t wl_splitmix64_next(uint64_t* state);
float wl_normal(uint64_t key, uint64_t i);
uint16_t wl_bf16(float f);
/* out[i] = bf16(normal(key(seed,stream), start+i) * col_scale[(start+i)%ncols] * scale);
 * col_scale may be NULL.  Host memory; nthreads host threads. */
void wl_fill_normal_bf16(uint64_t seed, uint64_t stream, uint64_t start, uint64_t n, float scale,
                         const float* col_scale, uint32_t ncols, uint16_t* out, int nthreads);
void wl_fill_normal_f32(uint64_t seed, uint64_t stream, uint64_t start, uint64_t n, float* out);
void wl_fill_u32(uint64_t seed, uint64_t stream, uint64_t start, uint64_t n, uint32_t* out);
void wl_permutation(uint64_t seed, uint64_t stream, int64_t n, int32_t* out);

/* ---- device library (libcsa2_workload_cuda.so) ----
 * Batched fill on the GPU: batch b draws from stream stream0 + b*stream_stride,
 * elements start .. start+per_batch-1, into out[b*per_batch + j] (device
 * memory, bf16 bits).  col_scale is a device array of ncols floats or NULL.
 * Asynchronous on `stream`.  Returns 0 on success, 1 on a bad argument,
 * 2 if the launch failed. */
#ifdef __CUDACC__
int wl_cuda_fill_normal_bf16(uint64_t seed, uint64_t stream0, uint64_t stream_stride,
                             int64_t nbatch, uint64_t per_batch, uint64_t start, float scale,
                             const float* col_scale, uint32_t ncols, uint16_t* out,
                             cudaStream_t stream);
#else
int wl_cuda_fill_normal_bf16(uint64_t seed, uint64_t stream0, uint64_t stream_stride,
                             int64_t nbatch, uint64_t per_batch, uint64_t start, float scale,
                             const float* col_scale, uint32_t ncols, uint16_t* out,
                             void* stream);
#endif

#ifdef __cplusplus
}
#endif

#endif /* CSA2_WORKLOAD_H */
