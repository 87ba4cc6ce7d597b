/*
 * Seeded synthetic attention inputs (q, k, v) as bf16 bit patterns.
 *
 * This module holds no attention arithmetic. It only turns (seed, tensor id,
 * flat element index) into a normal sample, multiplies it by an optional
 * per-head and per-channel factor, and rounds the product to bf16
 * (round-to-nearest-even). Both the CUDA path and the CPU oracle consume the
 * bytes it writes, so the two sides always see identical inputs.
 *
 * Generator, in published terms:
 *   - splitmix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014; the 64-bit finaliser as popularised by
 *     Vigna) keyed per stream: key = mix(mix(seed) ^ mix(tensor_id + 1)),
 *     draw for pair p = mix(key + p).
 *   - Box-Muller transform (Box & Muller, 1958) on the two 32-bit halves of a
 *     draw: u1 from the high half, u2 from the low half, both mapped to the
 *     open interval (0, 1) as (x + 0.5) / 2^32. Element 2p takes
 *     r*cos(2*pi*u2), element 2p+1 takes r*sin(2*pi*u2), r = sqrt(-2 ln u1).
 *   - value = bf16_rne((float)(z * head_scale[h] * chan_scale[h*D + d])).
 *
 * The flat element index is the row-major index into a [B, N, H, D] tensor,
 * so the same (seed, tensor id) always yields the same value at the same
 * (b, n, h, d), independent of how the fill is split across threads.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define TM_INPUTS_MAX_THREADS 256

static inline uint64_t mix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

uint64_t tm_inputs_stream_key(uint64_t seed, int tensor_id) {
  return mix64(mix64(seed) ^ mix64((uint64_t)tensor_id + 1ULL));
}

/* Normal sample number n of the stream with the given key. */
double tm_inputs_normal_at(uint64_t key, uint64_t n) {
  uint64_t x = mix64(key + (n >> 1));
  double u1 = ((double)(x >> 32) + 0.5) * (1.0 / 4294967296.0);
  double u2 = ((double)(x & 0xFFFFFFFFULL) + 0.5) * (1.0 / 4294967296.0);
  double r = sqrt(-2.0 * log(u1));
  double a = 6.283185307179586476925286766559 * u2;
  return (n & 1ULL) ? r * sin(a) : r * cos(a);
}

typedef struct {
  uint16_t* out;
  uint64_t begin, end;  /* flat element range [begin, end) */
  uint64_t key;
  int H, D;
  const float* head_scale;
  const float* chan_scale;
} fill_job;

static void* fill_worker(void* arg) {
  fill_job* j = (fill_job*)arg;
  const uint64_t HD = (uint64_t)j->H * (uint64_t)j->D;
  uint64_t n = j->begin;
  while (n < j->end) {
    uint64_t x = mix64(j->key + (n >> 1));
    double u1 = ((double)(x >> 32) + 0.5) * (1.0 / 4294967296.0);
    double u2 = ((double)(x & 0xFFFFFFFFULL) + 0.5) * (1.0 / 4294967296.0);
    double r = sqrt(-2.0 * log(u1));
    double a = 6.283185307179586476925286766559 * u2;
    double zz[2] = {r * cos(a), r * sin(a)};
    uint64_t first = n, last = (n | 1ULL) + 1ULL; /* this draw covers elements 2p, 2p+1 */
    if (last > j->end) last = j->end;
    for (uint64_t e = first; e < last; ++e) {
      uint64_t hd = e % HD;
      int h = (int)(hd / (uint64_t)j->D);
      double s = 1.0;
      if (j->head_scale) s *= (double)j->head_scale[h];
      if (j->chan_scale) s *= (double)j->chan_scale[hd];
      j->out[e] = f32_to_bf16_rne((float)(zz[e & 1ULL] * s));
    }
    n = last;
  }
  return NULL;
}

/*
 * Fill out[B*N*H*D] (bf16 bit patterns) for a [B, N, H, D] tensor.
 * head_scale: H floats or NULL. chan_scale: H*D floats or NULL.
 * Returns 0 on success, -1 on a bad argument.
 */
int tm_inputs_fill_bf16(uint16_t* out, long long B, long long N, int H, int D, uint64_t seed,
                        int tensor_id, const float* head_scale, const float* chan_scale,
                        int nthreads) {
  if (!out || B < 0 || N < 0 || H < 1 || D < 1) return -1;
  uint64_t total = (uint64_t)B * (uint64_t)N * (uint64_t)H * (uint64_t)D;
  if (total == 0) return 0;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > TM_INPUTS_MAX_THREADS) nthreads = TM_INPUTS_MAX_THREADS;
  uint64_t key = tm_inputs_stream_key(seed, tensor_id);
  fill_job jobs[TM_INPUTS_MAX_THREADS];
  pthread_t th[TM_INPUTS_MAX_THREADS];
  /* split on even boundaries so no Box-Muller pair straddles two threads */
  uint64_t chunk = ((total / (uint64_t)nthreads) + 2ULL) & ~1ULL;
  int used = 0;
  for (int t = 0; t < nthreads; ++t) {
    uint64_t b = (uint64_t)t * chunk;
    if (b >= total) break;
    uint64_t e = b + chunk < total ? b + chunk : total;
    jobs[t].out = out; jobs[t].begin = b; jobs[t].end = e; jobs[t].key = key;
    jobs[t].H = H; jobs[t].D = D; jobs[t].head_scale = head_scale; jobs[t].chan_scale = chan_scale;
    used = t + 1;
  }
  int started = 0;
  for (int t = 1; t < used; ++t) {
    if (pthread_create(&th[t], NULL, fill_worker, &jobs[t]) != 0) break;
    started = t;
  }
  fill_worker(&jobs[0]);
  for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
  for (int t = started + 1; t < used; ++t) fill_worker(&jobs[t]); /* threads that failed to start */
  return 0;
}
