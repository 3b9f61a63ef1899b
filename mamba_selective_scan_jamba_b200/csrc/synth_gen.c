/* Seeded synthetic-input generator (host code, no mixer arithmetic).
 *
 * SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): draw i of a stream with
 * seed s is mix(s + (i + 1) * 0x9E3779B97F4A7C15).  Uniform doubles keep the
 * top 53 bits; normals use Box-Muller on the pair of uniforms (2k, 2k+1):
 * r = sqrt(-2 log1p(-u0)), values r cos(2 pi u1) and r sin(2 pi u1).
 * Outputs can be written as float64, float32, or bf16 bit patterns (float32
 * first, then round to nearest even on the upper 16 bits).
 *
 * Work is split over threads by index ranges; every value depends only on
 * (seed, index), so the result is the same for any thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>
#include <unistd.h>

static inline uint64_t sm_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline double sm_uniform(uint64_t seed, int64_t i) {
  uint64_t z = sm_mix(seed + (uint64_t)(i + 1) * 0x9E3779B97F4A7C15ULL);
  return (double)(z >> 11) * (1.0 / 9007199254740992.0);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
  return (uint16_t)u;
}

enum { OUT_F64 = 0, OUT_F32 = 1, OUT_BF16 = 2 };

typedef struct {
  uint64_t seed;
  int64_t start, lo, hi;  /* fill out[lo..hi) with draws start+lo .. */
  double scale, shift;
  int kind;               /* 0 uniform, 1 normal */
  int out_type;
  void* out;
} job_t;

static void put(job_t* j, int64_t k, double v) {
  v = v * j->scale + j->shift;
  if (j->out_type == OUT_F64) ((double*)j->out)[k] = v;
  else if (j->out_type == OUT_F32) ((float*)j->out)[k] = (float)v;
  else ((uint16_t*)j->out)[k] = f32_to_bf16_rne((float)v);
}

static void* run_job(void* arg) {
  job_t* j = (job_t*)arg;
  const double two_pi = 6.283185307179586476925286766559;
  if (j->kind == 0) {
    for (int64_t k = j->lo; k < j->hi; ++k) put(j, k, sm_uniform(j->seed, j->start + k));
  } else {
    /* start is even; pair p covers draws (2p, 2p+1) of the stream */
    int64_t k = j->lo;
    while (k < j->hi) {
      int64_t g = j->start + k;
      int64_t p0 = g & ~(int64_t)1;
      double u0 = sm_uniform(j->seed, p0), u1 = sm_uniform(j->seed, p0 + 1);
      double r = sqrt(-2.0 * log1p(-u0));
      double v = (g & 1) ? r * sin(two_pi * u1) : r * cos(two_pi * u1);
      put(j, k, v);
      ++k;
    }
  }
  return 0;
}

static void fill(uint64_t seed, int64_t start, int64_t n, double scale, double shift,
                 int kind, int out_type, void* out, int threads) {
  if (n <= 0) return;
  if (threads <= 0) {
    long c = sysconf(_SC_NPROCESSORS_ONLN);
    threads = c > 0 ? (int)c : 1;
    if (threads > 64) threads = 64;
  }
  if (n < (1 << 16)) threads = 1;
  job_t jobs[64];
  pthread_t th[64];
  int64_t per = (n + threads - 1) / threads;
  int used = 0;
  for (int t = 0; t < threads; ++t) {
    int64_t lo = (int64_t)t * per, hi = lo + per > n ? n : lo + per;
    if (lo >= hi) break;
    jobs[t] = (job_t){seed, start, lo, hi, scale, shift, kind, out_type, out};
    used++;
  }
  for (int t = 1; t < used; ++t) pthread_create(&th[t], 0, run_job, &jobs[t]);
  run_job(&jobs[0]);
  for (int t = 1; t < used; ++t) pthread_join(th[t], 0);
}

/* out[k] = scale * U(start + k) + shift */
void jms_uniform(uint64_t seed, int64_t start, int64_t n, double scale, double shift,
                 int out_type, void* out, int threads) {
  fill(seed, start, n, scale, shift, 0, out_type, out, threads);
}

/* out[k] = scale * Normal(start + k) + shift */
void jms_normal(uint64_t seed, int64_t start, int64_t n, double scale, double shift,
                int out_type, void* out, int threads) {
  fill(seed, start, n, scale, shift, 1, out_type, out, threads);
}
