/*
 * Seeded, counter-based input generator for the MoE-layer workloads.
 *
 * This file holds NO arithmetic of the method (no routing, no expert FFN, no
 * softmax); it only turns (seed, stream, element index) into numbers. Both the
 * CPU oracle's tests and the GPU path draw their inputs from it, so the two
 * sides see bit-identical operands.
 *
 * Definition (the whole generator):
 *   key(seed, stream) = mix(mix(seed) ^ (stream * 0xD1B54A32D192ED03 + 0x8CB92BA72F3D8DD7))
 *   u64(key, i)       = mix(key + (i + 1) * 0x9E3779B97F4A7C15)          (SplitMix64's i-th output)
 *   mix(z)            = SplitMix64 finaliser (Steele, Lea, Flood 2014):
 *                         z = (z ^ z>>30) * 0xBF58476D1CE4E5B9
 *                         z = (z ^ z>>27) * 0x94D049BB133111EB
 *                         z ^ z>>31
 *   normal element 2j, 2j+1 = Box-Muller (1958) of r = u64(key, j):
 *       u1 = (hi32(r) + 0.5) / 2^32,  u2 = (lo32(r) + 0.5) / 2^32
 *       z0 = sqrt(-2 ln u1) cos(2 pi u2),   z1 = sqrt(-2 ln u1) sin(2 pi u2)
 *   value = std * z, in double, rounded to fp32 (round-to-nearest-even) and,
 *   for bf16 outputs, the fp32 value rounded again to bf16 (nearest-even).
 *   permutation(m) = Fisher-Yates: for i = m-1 .. 1, swap(p[i], p[u64(key, i) mod (i+1)]).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

uint64_t gen_stream_key(uint64_t seed, uint64_t stream) {
  return mix64(mix64(seed) ^ (stream * 0xD1B54A32D192ED03ULL + 0x8CB92BA72F3D8DD7ULL));
}

uint64_t gen_u64(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * 0x9E3779B97F4A7C15ULL); }

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t b;
  memcpy(&b, &f, 4);
  uint32_t lsb = (b >> 16) & 1u;
  b += 0x7FFFu + lsb;
  return (uint16_t)(b >> 16);
}

static inline void normal_pair(uint64_t key, uint64_t j, double* z0, double* z1) {
  uint64_t r = gen_u64(key, j);
  double u1 = ((double)(r >> 32) + 0.5) * (1.0 / 4294967296.0);
  double u2 = ((double)(r & 0xFFFFFFFFULL) + 0.5) * (1.0 / 4294967296.0);
  double rad = sqrt(-2.0 * log(u1));
  double th = 6.283185307179586476925 * u2;
  *z0 = rad * cos(th);
  *z1 = rad * sin(th);
}

/* dtype: 0 = fp32, 1 = bf16 (raw bits). */
static void fill_range(uint64_t key, double stdv, int dtype, void* out, int64_t lo, int64_t hi) {
  for (int64_t i = lo; i < hi; ++i) {
    double z0, z1;
    normal_pair(key, (uint64_t)(i >> 1), &z0, &z1);
    float v = (float)(stdv * ((i & 1) ? z1 : z0));
    if (dtype == 0)
      ((float*)out)[i] = v;
    else
      ((uint16_t*)out)[i] = f32_to_bf16_rne(v);
  }
}

typedef struct {
  uint64_t key;
  double stdv;
  int dtype;
  void* out;
  int64_t lo, hi;
} fill_job_t;

static void* fill_worker(void* p) {
  fill_job_t* j = (fill_job_t*)p;
  fill_range(j->key, j->stdv, j->dtype, j->out, j->lo, j->hi);
  return 0;
}

/* Fill out[0..n) with std * N(0,1) from stream (seed, stream). Returns 0 on success. */
int gen_normal(uint64_t seed, uint64_t stream, double stdv, int dtype, void* out, int64_t n, int nthreads) {
  if (n <= 0) return 0;
  if (dtype != 0 && dtype != 1) return 1;
  uint64_t key = gen_stream_key(seed, stream);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < 65536 || nthreads == 1) {
    fill_range(key, stdv, dtype, out, 0, n);
    return 0;
  }
  pthread_t th[256];
  int running[256];
  fill_job_t jobs[256];
  int64_t chunk = (n + nthreads - 1) / nthreads;
  chunk = (chunk + 1) & ~(int64_t)1;
  for (int t = 0; t < nthreads; ++t) {
    running[t] = 0;
    int64_t lo = (int64_t)t * chunk, hi = lo + chunk;
    if (lo >= n) continue;
    if (hi > n) hi = n;
    jobs[t] = (fill_job_t){key, stdv, dtype, out, lo, hi};
    if (pthread_create(&th[t], 0, fill_worker, &jobs[t]) == 0)
      running[t] = 1;
    else
      fill_range(key, stdv, dtype, out, lo, hi);
  }
  for (int t = 0; t < nthreads; ++t)
    if (running[t]) pthread_join(th[t], 0);
  return 0;
}

/* Seeded Fisher-Yates permutation of 0..m-1. */
int gen_permutation(uint64_t seed, uint64_t stream, int32_t m, int32_t* out) {
  if (m <= 0) return 1;
  uint64_t key = gen_stream_key(seed, stream);
  for (int32_t i = 0; i < m; ++i) out[i] = i;
  for (int32_t i = m - 1; i >= 1; --i) {
    int32_t j = (int32_t)(gen_u64(key, (uint64_t)i) % (uint64_t)(i + 1));
    int32_t t = out[i];
    out[i] = out[j];
    out[j] = t;
  }
  return 0;
}
