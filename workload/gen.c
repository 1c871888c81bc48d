/*
 * Seeded synthetic-input generator, host side (plain C, no method arithmetic).
 *
 * Every input of the CSA2 workloads (KV rows, indexer keys, queries, page
 * permutations, lengths, miss flags) is drawn from one counter-based stream
 * built on SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014; finaliser constants as in Vigna's public
 * splitmix64.c).  A value is a pure function of (seed, stream, index), so
 * any row of any sequence can be regenerated on its own, and the CUDA twin
 * of this file (gen_device.cu) produces bit-identical values on the GPU.
 *
 * Definitions (shared with gen_device.cu, checked against each other by the
 * GPU tests):
 *   mix64(z)        = SplitMix64 output finaliser
 *   key(seed, s)    = mix64(seed ^ mix64(s + GAMMA))
 *   u64(key, i)     = mix64(key + (i + 1) * GAMMA)           (mod 2^64)
 *   normal(key, i)  = (S - 6*2^24) * 2^-24, S = sum of the twelve 24-bit
 *                     fields (bits 40..63 and 16..39) of u64(key, 6i+j),
 *                     j = 0..5; S - 6*2^24 is converted to float once with
 *                     round-to-nearest-even (Irwin-Hall(12) approximation of
 *                     N(0,1), exact integer arithmetic up to that one rounding)
 *   bf16(x)         = round-to-nearest-even of an fp32 value to bfloat16
 */
#include <stdint.h>
#include <string.h>
#include <pthread.h>

#define WL_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t wl_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

uint64_t wl_key(uint64_t seed, uint64_t stream) {
  return wl_mix64(seed ^ wl_mix64(stream + WL_GAMMA));
}

uint64_t wl_u64(uint64_t key, uint64_t i) { return wl_mix64(key + (i + 1) * WL_GAMMA); }

/* First output of a plain SplitMix64 generator started at `state`; used only
 * to pin the finaliser against the published reference sequence. */
uint64_t wl_splitmix64_next(uint64_t* state) {
  *state += WL_GAMMA;
  return wl_mix64(*state);
}

float wl_normal(uint64_t key, uint64_t i) {
  int32_t s = 0;
  for (int j = 0; j < 6; ++j) {
    uint64_t h = wl_u64(key, 6 * i + (uint64_t)j);
    s += (int32_t)(h >> 40) + (int32_t)((h >> 16) & 0xFFFFFFu);
  }
  s -= 6 << 24; /* |s| < 6*2^24 < 2^27: exact in int32 */
  return (float)s * 0x1p-24f;
}

uint16_t wl_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* ---- bulk fills, split over host threads ---- */

typedef struct {
  uint64_t key, start, lo, hi;
  float scale;
  const float* col_scale;
  uint32_t ncols;
  uint16_t* out;
} wl_job;

static void* wl_fill_worker(void* p) {
  wl_job* j = (wl_job*)p;
  for (uint64_t i = j->lo; i < j->hi; ++i) {
    uint64_t e = j->start + i;
    float v = wl_normal(j->key, e);
    if (j->col_scale) v = v * j->col_scale[e % j->ncols];
    v = v * j->scale;
    j->out[i] = wl_bf16(v);
  }
  return NULL;
}

/* out[i] = bf16( normal(key(seed,stream), start+i) * col_scale[(start+i) % ncols] * scale )
 * (col_scale may be NULL; the two multiplies are fp32 and happen in that order). */
void wl_fill_normal_bf16(uint64_t seed, uint64_t stream, uint64_t start, uint64_t n, float scale,
                         const float* col_scale, uint32_t ncols, uint16_t* out, int nthreads) {
  uint64_t key = wl_key(seed, stream);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 64) nthreads = 64;
  if (n < 65536) nthreads = 1;
  wl_job jobs[64];
  pthread_t th[64];
  for (int t = 0; t < nthreads; ++t) {
    jobs[t].key = key;
    jobs[t].start = start;
    jobs[t].lo = n * (uint64_t)t / (uint64_t)nthreads;
    jobs[t].hi = n * (uint64_t)(t + 1) / (uint64_t)nthreads;
    jobs[t].scale = scale;
    jobs[t].col_scale = col_scale;
    jobs[t].ncols = ncols ? ncols : 1;
    jobs[t].out = out;
  }
  if (nthreads == 1) {
    wl_fill_worker(&jobs[0]);
    return;
  }
  for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, wl_fill_worker, &jobs[t]);
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
}

/* out[i] = normal(key(seed,stream), start+i) as fp32 (before any bf16 rounding). */
void wl_fill_normal_f32(uint64_t seed, uint64_t stream, uint64_t start, uint64_t n, float* out) {
  uint64_t key = wl_key(seed, stream);
  for (uint64_t i = 0; i < n; ++i) out[i] = wl_normal(key, start + i);
}

/* out[i] = top 32 bits of u64(key(seed,stream), start+i). */
void wl_fill_u32(uint64_t seed, uint64_t stream, uint64_t start, uint64_t n, uint32_t* out) {
  uint64_t key = wl_key(seed, stream);
  for (uint64_t i = 0; i < n; ++i) out[i] = (uint32_t)(wl_u64(key, start + i) >> 32);
}

/* Fisher-Yates permutation of 0..n-1; step t (t = 0..n-2) swaps slot i = n-1-t
 * with j = floor(r * (i+1) / 2^32), r = top 32 bits of u64(key, t). */
void wl_permutation(uint64_t seed, uint64_t stream, int64_t n, int32_t* out) {
  uint64_t key = wl_key(seed, stream);
  for (int64_t i = 0; i < n; ++i) out[i] = (int32_t)i;
  for (int64_t i = n - 1, t = 0; i > 0; --i, ++t) {
    uint64_t r = wl_u64(key, (uint64_t)t) >> 32;
    int64_t j = (int64_t)((r * (uint64_t)(i + 1)) >> 32);
    int32_t tmp = out[i];
    out[i] = out[j];
    out[j] = tmp;
  }
}
