/*
 * Seeded synthetic inputs for the MXFP4 MoE layer.
 *
 * This file holds no step of the layer's arithmetic: it only draws the
 * random inputs (activations, router logits, bf16 expert weights) that both
 * the CUDA library's tests/benchmark and the CPU oracle consume.
 *
 * Generator: counter-based splitmix64 (G. Steele, D. Lea, C. Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014).  Draw n of
 * stream `sid` under seed `seed` is mix(base(seed, sid) + (n+1)*GAMMA), so
 * any element can be produced independently of the others and the result
 * does not depend on how the work is split across threads.
 * Normal deviates: Box-Muller on a pair of 53-bit uniforms (draws 2p, 2p+1
 * give elements 2p and 2p+1 as the cosine and sine branch).
 * bf16 values are the round-to-nearest-even of the double-precision deviate
 * (times sigma), rounded once.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_base(uint64_t seed, uint64_t sid) {
  return mix64(mix64(seed + GAMMA) ^ (sid * 0xD1B54A32D192ED03ULL));
}

static inline uint64_t draw(uint64_t base, uint64_t n) {
  return mix64(base + (n + 1) * GAMMA);
}

/* uniform in [0, 1) with 53 random bits */
static inline double u01(uint64_t r) { return (double)(r >> 11) * 0x1.0p-53; }

static inline double normal_at(uint64_t base, uint64_t i) {
  const uint64_t p = i >> 1;
  const double u1 = ((double)(draw(base, 2 * p) >> 11) + 1.0) * 0x1.0p-53; /* (0,1] */
  const double u2 = u01(draw(base, 2 * p + 1));
  const double r = sqrt(-2.0 * log(u1));
  const double th = 6.283185307179586476925286766559 * u2;
  return (i & 1) ? r * sin(th) : r * cos(th);
}

/* round-to-nearest-even of a double onto bf16 (8 significant bits,
 * exponent range of fp32, subnormals kept, overflow to infinity) */
static uint16_t bf16_from_double(double x) {
  if (isnan(x)) return 0x7FC0;
  const uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e);            /* a = f * 2^e, f in [0.5, 1) -> floor(log2 a) = e-1 */
  int q = (e - 1) - 7;     /* quantum exponent for 8 significant bits */
  if (q < -133) q = -133;  /* bf16 subnormal quantum 2^-133 */
  double r = nearbyint(ldexp(a, -q)); /* default rounding mode: ties to even */
  r = ldexp(r, q);
  if (r >= 0x1.0p128) return sign | 0x7F80;
  float f = (float)r; /* exact: r has <= 8 significant bits in fp32 range */
  uint32_t bits;
  memcpy(&bits, &f, 4);
  return sign | (uint16_t)((bits >> 16) & 0x7FFF);
}

/* ---------------------------------------------------------------- jobs */

typedef struct {
  uint64_t base, mask_base;
  uint64_t offset;
  int64_t lo, hi;
  double sigma, p_out, factor;
  int kind; /* 0 = bf16 normal, 1 = bf16 normal with outliers, 2 = uniform f64 */
  uint16_t* out16;
  double* out64;
} job_t;

static void* run_job(void* arg) {
  job_t* j = (job_t*)arg;
  for (int64_t n = j->lo; n < j->hi; ++n) {
    const uint64_t i = j->offset + (uint64_t)n;
    if (j->kind == 2) {
      j->out64[n] = u01(draw(j->base, i));
      continue;
    }
    double v = j->sigma * normal_at(j->base, i);
    if (j->kind == 1 && u01(draw(j->mask_base, i)) < j->p_out) v *= j->factor;
    j->out16[n] = bf16_from_double(v);
  }
  return NULL;
}

static void run_parallel(job_t proto, int64_t n, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < 65536) nthreads = 1;
  pthread_t th[256];
  job_t jobs[256];
  int created[256];
  const int64_t chunk = (n + nthreads - 1) / nthreads;
  int used = 0;
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = proto;
    jobs[t].lo = (int64_t)t * chunk;
    jobs[t].hi = jobs[t].lo + chunk < n ? jobs[t].lo + chunk : n;
    if (jobs[t].lo >= jobs[t].hi) break;
    created[t] = pthread_create(&th[t], NULL, run_job, &jobs[t]) == 0;
    if (!created[t]) run_job(&jobs[t]);
    used = t + 1;
  }
  for (int t = 0; t < used; ++t)
    if (created[t]) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------------- exports */

/* out[n] = bf16(sigma * N(0,1) draw (offset+n) of stream sid), n < count */
void syn_normal_bf16(uint64_t seed, uint64_t sid, uint64_t offset, int64_t count,
                     double sigma, uint16_t* out, int nthreads) {
  job_t j;
  memset(&j, 0, sizeof j);
  j.base = stream_base(seed, sid);
  j.offset = offset;
  j.sigma = sigma;
  j.kind = 0;
  j.out16 = out;
  run_parallel(j, count, nthreads);
}

/* as syn_normal_bf16, but an independent Bernoulli(p_out) mask drawn from
 * stream mask_sid multiplies the double-precision value by `factor` before
 * the single rounding to bf16 */
void syn_normal_outliers_bf16(uint64_t seed, uint64_t sid, uint64_t mask_sid,
                              uint64_t offset, int64_t count, double sigma,
                              double p_out, double factor, uint16_t* out,
                              int nthreads) {
  job_t j;
  memset(&j, 0, sizeof j);
  j.base = stream_base(seed, sid);
  j.mask_base = stream_base(seed, mask_sid);
  j.offset = offset;
  j.sigma = sigma;
  j.p_out = p_out;
  j.factor = factor;
  j.kind = 1;
  j.out16 = out;
  run_parallel(j, count, nthreads);
}

/* out[n] = N(0,1) draw (offset+n) of stream sid as double (no rounding) */
void syn_normal_f64(uint64_t seed, uint64_t sid, uint64_t offset, int64_t count,
                    double* out) {
  const uint64_t base = stream_base(seed, sid);
  for (int64_t n = 0; n < count; ++n) out[n] = normal_at(base, offset + (uint64_t)n);
}

/* out[n] = uniform [0,1) draw (offset+n) of stream sid */
void syn_uniform_f64(uint64_t seed, uint64_t sid, uint64_t offset, int64_t count,
                     double* out, int nthreads) {
  job_t j;
  memset(&j, 0, sizeof j);
  j.base = stream_base(seed, sid);
  j.offset = offset;
  j.kind = 2;
  j.out64 = out;
  run_parallel(j, count, nthreads);
}

/* router logits [T][E] as fp32: N(0,1) draw (t*E+e) of stream sid plus an
 * optional per-expert bias (double, may be NULL), rounded once to fp32 */
void syn_logits_f32(uint64_t seed, uint64_t sid, int64_t T, int64_t E,
                    const double* bias, float* out) {
  const uint64_t base = stream_base(seed, sid);
  for (int64_t t = 0; t < T; ++t)
    for (int64_t e = 0; e < E; ++e) {
      double v = normal_at(base, (uint64_t)(t * E + e));
      if (bias) v += bias[e];
      out[t * E + e] = (float)v;
    }
}

/* the bf16 rounding used above, exposed for the generator's own tests */
uint16_t syn_bf16_from_double(double x) { return bf16_from_double(x); }
