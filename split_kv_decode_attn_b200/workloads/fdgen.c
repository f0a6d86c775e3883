/*
 * fdgen.c — seeded, counter-based input generator for the decode-attention
 * workloads.  It holds none of the attention arithmetic: it only draws the
 * numbers that the test harness, the benchmark and the oracle all take as
 * input, so that both sides of a parity check see the same bytes.
 *
 * Definition (portable, random-access):
 *   SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
 *   generators", OOPSLA 2014; constants as published by Vigna):
 *     x_i  = seed + (i + 1) * 0x9E3779B97F4A7C15          (mod 2^64)
 *     u64_i = mix(x_i), mix(z) = z ^= z>>30, z *= 0xBF58476D1CE4E5B9,
 *                                z ^= z>>27, z *= 0x94D049BB133111EB,
 *                                z ^= z>>31
 *   Standard normal from one 64-bit draw (Box-Muller, cosine branch):
 *     u1 = (hi32 + 0.5) / 2^32,  u2 = (lo32 + 0.5) / 2^32     (both in (0,1))
 *     z  = sqrt(-2 ln u1) * cos(2 pi u2)                       (double)
 *   bf16 value: z rounded to fp32 (round-to-nearest-even), then the fp32
 *   rounded to bf16 (round-to-nearest-even on the upper 16 bits).
 *
 * Build: gcc -O2 -shared -fPIC -pthread fdgen.c -o libfdgen.so -lm
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define FDGEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t fdgen_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Output i of the SplitMix64 stream started at `seed`. */
static inline uint64_t fdgen_at(uint64_t seed, uint64_t i) {
  return fdgen_mix(seed + (i + 1) * FDGEN_GAMMA);
}

static inline uint16_t fdgen_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  /* z is finite by construction; round to nearest, ties to even */
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static inline double fdgen_normal(uint64_t r) {
  const double inv32 = 1.0 / 4294967296.0;
  double u1 = ((double)(r >> 32) + 0.5) * inv32;
  double u2 = ((double)(r & 0xFFFFFFFFu) + 0.5) * inv32;
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

/* Raw 64-bit draws i = offset .. offset+n-1 of stream `seed`. */
void fdgen_u64(uint64_t seed, uint64_t offset, uint64_t n, uint64_t* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = fdgen_at(seed, offset + i);
}

/* Standard normal draws as fp64 (used for small derived inputs). */
void fdgen_normal_f64(uint64_t seed, uint64_t offset, uint64_t n, double* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = fdgen_normal(fdgen_at(seed, offset + i));
}

typedef struct {
  uint64_t seed, offset, begin, end;
  uint16_t* out;
} fdgen_job;

static void* fdgen_worker(void* arg) {
  fdgen_job* j = (fdgen_job*)arg;
  for (uint64_t i = j->begin; i < j->end; ++i)
    j->out[i] = fdgen_f32_to_bf16((float)fdgen_normal(fdgen_at(j->seed, j->offset + i)));
  return 0;
}

/* bf16 bit patterns of N(0,1) draws i = offset .. offset+n-1, split over
 * `nthreads` POSIX threads (the result does not depend on the thread count). */
int fdgen_normal_bf16(uint64_t seed, uint64_t offset, uint64_t n, uint16_t* out,
                      int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((uint64_t)nthreads > n / 65536 + 1) nthreads = (int)(n / 65536 + 1);
  pthread_t th[256];
  int joined[256];
  fdgen_job jobs[256];
  uint64_t per = (n + (uint64_t)nthreads - 1) / (uint64_t)nthreads;
  for (int t = 0; t < nthreads; ++t) {
    uint64_t b = per * (uint64_t)t, e = b + per;
    if (b > n) b = n;
    if (e > n) e = n;
    jobs[t].seed = seed;
    jobs[t].offset = offset;
    jobs[t].begin = b;
    jobs[t].end = e;
    jobs[t].out = out;
    joined[t] = 0;
    if (t == 0) continue;
    if (pthread_create(&th[t], 0, fdgen_worker, &jobs[t]) != 0)
      fdgen_worker(&jobs[t]); /* run inline if a thread cannot start */
    else
      joined[t] = 1;
  }
  fdgen_worker(&jobs[0]);
  for (int t = 1; t < nthreads; ++t)
    if (joined[t]) pthread_join(th[t], 0);
  return 0;
}
