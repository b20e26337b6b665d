/*
 * oracle.c -- plain, slow, double-precision CPU restatement of the MXFP4
 * Mixture-of-Experts layer.  TEST INFRASTRUCTURE ONLY: it is the checker the
 * CUDA library is compared against; the library never calls, links or loads
 * it, and it shares no code, header or table with the library.
 *
 * Sources (web pages, cited by title and section):
 *  [P1] "Tricks from OpenAI gpt-oss you can use with transformers" (Korean
 *       summary), section 6 (MXFP4 format: E2M1 elements, one shared scale
 *       per 32-element block) and section 8 (kernels must honour the blocks
 *       and their scales inside GEMMs).
 *  [P2] "Welcome GPT OSS, the new open-source model family from OpenAI"
 *       (Korean summary), section 4 (token-choice MoE, SwiGLU,
 *       softmax-after-topk).
 *  [P3] aitrends.kr talk summary, chapters "Architecture details" (4 active
 *       experts of 32/128), "Hardware optimisation" (weights kept low
 *       precision, raised only for compute) and "Q&A" (independent experts,
 *       no shared expert).
 *  [P4] "MXFP4-based MoE technical review", section 1 (MXFP4 is the OCP
 *       Microscaling format: E8M0 power-of-two shared scale).
 *  [P5] agentlenshq "Transformers ... GPT-OSS" (Japanese), section "What is
 *       MXFP4" (1 sign, 2 exponent, 1 mantissa bit; 32-element blocks).
 * Readings where the pages are silent (each is listed in the design notes):
 *  - scale byte = floor(log2 amax) - 2 + 127 via the bf16 exponent field,
 *    clamped to [0, 254]; zero / subnormal amax gives byte 0;
 *  - element code: round to nearest, ties to the even mantissa bit, onto
 *    {0,0.5,1,1.5,2,3,4,6}, saturating at 6, sign kept (so -0 is code 8);
 *  - element 2i in the low nibble, 2i+1 in the high nibble;
 *  - SwiGLU is silu(gate) * up with no clamp, bias or offset; gate rows come
 *    first in the [2F][D] gate/up matrix;
 *  - h, y and out are rounded to bf16 (round to nearest even) exactly where
 *    the library hands them over as bf16; all else is exact or fp64;
 *  - top-k order: logit descending, expert index ascending on ties;
 *  - the combine sums the k terms in ascending j.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------ bf16 <-> double */

/* exact value of a bf16 bit pattern */
double oracle_bf16_value(uint16_t b) {
  uint32_t bits = (uint32_t)b << 16;
  float f;
  memcpy(&f, &bits, 4);
  return (double)f;
}

/* round a double to the nearest bf16, ties to even; bf16 keeps 8 significant
 * bits with the fp32 exponent range (subnormal quantum 2^-133); values that
 * round to 2^128 or beyond become infinity */
uint16_t oracle_bf16_round(double x) {
  if (isnan(x)) return 0x7FC0;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (a == 0.0) return sign;
  if (isinf(a)) return sign | 0x7F80;
  int e;
  frexp(a, &e);        /* a in [2^(e-1), 2^e) */
  int q = e - 8;       /* 8 significant bits: quantum 2^(e-1-7) */
  if (q < -133) q = -133;
  double m = ldexp(a, -q);   /* exact */
  double fl = floor(m);
  double rem = m - fl;
  double r;
  if (rem > 0.5) r = fl + 1.0;
  else if (rem < 0.5) r = fl;
  else r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0; /* tie: to even */
  double v = ldexp(r, q);
  if (v >= 0x1.0p128) return sign | 0x7F80;
  float f = (float)v; /* exact */
  uint32_t bits;
  memcpy(&bits, &f, 4);
  return sign | (uint16_t)((bits >> 16) & 0x7FFF);
}

/* ------------------------------------------------------------------- MXFP4 */

/* magnitudes of the eight E2M1 codes (sign bit excluded) [P1 s6, P5] */
static const double E2M1_MAGNITUDE[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* value of one 4-bit code under scale byte b: sign * magnitude * 2^(b-127) */
double oracle_mxfp4_value(uint8_t code, uint8_t scale_byte) {
  double mag = E2M1_MAGNITUDE[code & 7];
  double v = (code & 8) ? -mag : mag;
  if (scale_byte == 255) return NAN; /* E8M0 NaN encoding; never produced */
  return ldexp(v, (int)scale_byte - 127);
}

/* E8M0 scale byte of one 32-element block [P4 s1; rule: floor(log2 amax)-2] */
static uint8_t block_scale_byte(const uint16_t* blk) {
  uint16_t amax_bits = 0;
  double amax = 0.0;
  for (int i = 0; i < 32; ++i) {
    double a = fabs(oracle_bf16_value(blk[i]));
    if (a > amax) {
      amax = a;
      amax_bits = blk[i] & 0x7FFF;
    }
  }
  if (amax == 0.0) return 0;
  int bexp = (amax_bits >> 7) & 0xFF; /* biased exponent of amax */
  int b = bexp - 2;                    /* floor(log2 amax) - 2 + 127 */
  if (b < 0) b = 0;
  if (b > 254) b = 254;
  return (uint8_t)b;
}

/* nearest E2M1 magnitude code to v >= 0, ties to the even mantissa bit,
 * saturating at 6.0 */
static uint8_t e2m1_magnitude_code(double v) {
  if (v <= 0.25) return 0;  /* 0.25 ties between 0 and 0.5 -> 0 (even) */
  if (v < 0.75) return 1;   /* 0.75 ties between 0.5 and 1 -> 1.0     */
  if (v <= 1.25) return 2;  /* 1.25 ties between 1 and 1.5 -> 1.0     */
  if (v < 1.75) return 3;   /* 1.75 ties between 1.5 and 2 -> 2.0     */
  if (v <= 2.5) return 4;   /* 2.5 ties between 2 and 3 -> 2.0        */
  if (v < 3.5) return 5;    /* 3.5 ties between 3 and 4 -> 4.0        */
  if (v <= 5.0) return 6;   /* 5 ties between 4 and 6 -> 4.0          */
  return 7;                 /* (5, inf) -> 6.0, saturating            */
}

/* rows [r0, r1) of the quantiser below */
static int64_t quantize_rows(const uint16_t* w, int64_t r0, int64_t r1, int64_t K, uint8_t* q,
                             uint8_t* s) {
  int64_t bad = 0;
  const int64_t nb = K / 32;
  for (int64_t r = r0; r < r1; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const uint16_t* blk = w + r * K + b * 32;
      int nonfinite = 0;
      for (int i = 0; i < 32; ++i)
        if (((blk[i] >> 7) & 0xFF) == 0xFF) nonfinite = 1;
      bad += nonfinite;
      uint8_t sb = block_scale_byte(blk);
      s[r * nb + b] = sb;
      double scale = ldexp(1.0, (int)sb - 127);
      for (int i = 0; i < 32; i += 2) {
        uint8_t c[2];
        for (int h = 0; h < 2; ++h) {
          double x = oracle_bf16_value(blk[i + h]);
          uint8_t code = e2m1_magnitude_code(fabs(x) / scale);
          if (signbit(x)) code |= 8;
          c[h] = code;
        }
        q[r * (K / 2) + (b * 32 + i) / 2] = (uint8_t)(c[0] | (c[1] << 4));
      }
    }
  }
  return bad;
}

typedef struct {
  const uint16_t* w;
  int64_t r0, r1, K;
  uint8_t *q, *s;
  int64_t bad;
} quant_job;

static void* quant_run(void* arg) {
  quant_job* j = (quant_job*)arg;
  j->bad = quantize_rows(j->w, j->r0, j->r1, j->K, j->q, j->s);
  return NULL;
}

/* bf16 [rows][K] -> codes [rows][K/2] + scale bytes [rows][K/32], rows split
 * over threads (each row is independent).  Returns the number of blocks
 * holding a NaN or infinity (their bytes are not meaningful). */
int64_t oracle_mxfp4_quantize_mt(const uint16_t* w, int64_t rows, int64_t K, uint8_t* q,
                                 uint8_t* s, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (rows < 64) nthreads = 1;
  pthread_t th[256];
  quant_job jobs[256];
  int created[256];
  int64_t chunk = (rows + nthreads - 1) / nthreads;
  int used = 0;
  for (int t = 0; t < nthreads; ++t) {
    quant_job j = {w, t * chunk, (t + 1) * chunk < rows ? (t + 1) * chunk : rows, K, q, s, 0};
    jobs[t] = j;
    if (jobs[t].r0 >= jobs[t].r1) break;
    created[t] = pthread_create(&th[t], NULL, quant_run, &jobs[t]) == 0;
    if (!created[t]) quant_run(&jobs[t]);
    used = t + 1;
  }
  int64_t bad = 0;
  for (int t = 0; t < used; ++t) {
    if (created[t]) pthread_join(th[t], NULL);
    bad += jobs[t].bad;
  }
  return bad;
}

int64_t oracle_mxfp4_quantize(const uint16_t* w, int64_t rows, int64_t K, uint8_t* q,
                              uint8_t* s) {
  return quantize_rows(w, 0, rows, K, q, s);
}

/* codes + scales [rows][K] -> double values */
void oracle_mxfp4_decode(const uint8_t* q, const uint8_t* s, int64_t rows, int64_t K,
                         double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = q[r * (K / 2) + k / 2];
      uint8_t code = (k & 1) ? (byte >> 4) : (byte & 15);
      out[r * K + k] = oracle_mxfp4_value(code, s[r * (K / 32) + k / 32]);
    }
}

/* ------------------------------------- training-style quantiser [P4 s2, s4] */
/*
 * "MXFP4-based MoE technical review", sections 2 and 4: MXFP4 training keeps
 * its quality with stochastic rounding and a random Hadamard transform.  The
 * page names the two techniques and no more; the readings taken here are:
 *  - the transform acts on each 32-element block along K (the block that
 *    shares one scale): y = H (s . x), H the 32 x 32 Sylvester Hadamard
 *    matrix (+1/-1 entries, H[i][j] = (-1)^popcount(i & j)), unnormalised,
 *    s a random sign per position j of block column K/32 given by the caller
 *    (bit j of signs[block column] set = negate); (H diag(s)) times its
 *    transpose is 32 I, so a product of two operands that carry the same
 *    transform along K is 32 times the plain product;
 *  - y is the exact value of that sum (fp64 here; every test input keeps it
 *    exact: 32 bf16 terms whose exponents span far less than 40 binades);
 *  - stochastic rounding moves |y| / scale to one of its two neighbours on
 *    the E2M1 grid, the upper one with probability equal to the distance from
 *    the lower one over the gap, drawn as u < frac with u a 16-bit uniform;
 *    to keep it unbiased no element may clip, so with rounding stochastic the
 *    scale exponent is the smallest that brings amax to at most 6:
 *    byte = 127 + ceil(log2(amax / 6)), clamped to [0, 254];
 *  - uniforms: Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel random
 *    numbers: as easy as 1, 2, 3", SC 2011) keyed by the 64-bit seed; element
 *    n = r K + c of the call draws from the counter (n / 8 low word, n / 8
 *    high word, 0, 0), output word (n % 8) / 2, low half for even n;
 *  - a transformed element's sign bit is set only for y < 0 (an exact zero
 *    is code 0); without the transform the sign bit is that of x, as in the
 *    deterministic quantiser, which this one equals when no flag is set.
 */
#define ORACLE_QUANT_RHT 1u
#define ORACLE_QUANT_SR 2u

/* Philox4x32-10: ten rounds of the two 32 x 32 -> 64-bit products and the
 * word permutation, the key bumped by the two Weyl constants between rounds */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    uint64_t p0 = (uint64_t)0xD2511F53u * c0;
    uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
    uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
    uint32_t n1 = (uint32_t)p1;
    uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    uint32_t n3 = (uint32_t)p0;
    c0 = n0;
    c1 = n1;
    c2 = n2;
    c3 = n3;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

/* the 16-bit uniform of element n of a call keyed by seed */
uint32_t oracle_sr_uniform16(uint64_t seed, uint64_t n) {
  uint32_t ctr[4] = {(uint32_t)(n / 8), (uint32_t)((n / 8) >> 32), 0u, 0u};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t out[4];
  oracle_philox4x32_10(ctr, key, out);
  uint32_t word = out[(n % 8) / 2];
  return (n & 1) ? (word >> 16) : (word & 0xFFFFu);
}

/* y = H (s . x) of one 32-element block, summed over j ascending */
void oracle_rht32(const double* x, uint32_t sign_word, double* y) {
  for (int i = 0; i < 32; ++i) {
    double acc = 0.0;
    for (int j = 0; j < 32; ++j) {
      double xj = ((sign_word >> j) & 1u) ? -x[j] : x[j];
      acc += (__builtin_popcount((unsigned)(i & j)) & 1) ? -xj : xj;
    }
    y[i] = acc;
  }
}

/* stochastic rounding of v >= 0 onto the E2M1 magnitudes with the 16-bit
 * uniform u: the lower neighbour, or the upper one when u / 2^16 < frac */
uint8_t oracle_sr_code(double v, uint32_t u) {
  if (v >= 6.0) return 7; /* on the top magnitude (or above it, clipped) */
  int c = 0;
  while (E2M1_MAGNITUDE[c + 1] <= v) ++c; /* G[c] <= v < G[c + 1] */
  double frac = (v - E2M1_MAGNITUDE[c]) / (E2M1_MAGNITUDE[c + 1] - E2M1_MAGNITUDE[c]);
  return (uint8_t)(((double)u / 65536.0 < frac) ? c + 1 : c);
}

/* scale byte from the block maximum of |y|: floor(log2 amax) - 2 + 127, and
 * with stochastic rounding one more when amax / 2^(floor(log2 amax) - 2) > 6 */
static uint8_t scale_byte_of(double amax, int sr) {
  if (amax == 0.0) return 0;
  int e;
  double m = frexp(amax, &e); /* amax = m 2^e, m in [0.5, 1) */
  int b = (e - 1) - 2 + 127;
  if (sr && m > 0.75) b += 1; /* significand above 1.5: 4 * 1.5 = 6 */
  if (b < 0) b = 0;
  if (b > 254) b = 254;
  return (uint8_t)b;
}

static int64_t quantize_ex_rows(const uint16_t* w, int64_t r0, int64_t r1, int64_t K,
                                uint32_t flags, const uint32_t* signs, uint64_t seed, uint8_t* q,
                                uint8_t* s) {
  const int rht = (flags & ORACLE_QUANT_RHT) != 0, sr = (flags & ORACLE_QUANT_SR) != 0;
  const int64_t nb = K / 32;
  int64_t bad = 0;
  for (int64_t r = r0; r < r1; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const uint16_t* blk = w + r * K + b * 32;
      double x[32], y[32];
      int neg[32], nonfinite = 0;
      for (int i = 0; i < 32; ++i) {
        if (((blk[i] >> 7) & 0xFF) == 0xFF) nonfinite = 1;
        x[i] = oracle_bf16_value(blk[i]);
      }
      bad += nonfinite;
      if (rht) {
        oracle_rht32(x, signs[b], y);
        for (int i = 0; i < 32; ++i) neg[i] = y[i] < 0.0;
      } else {
        for (int i = 0; i < 32; ++i) {
          y[i] = x[i];
          neg[i] = signbit(x[i]) != 0;
        }
      }
      double amax = 0.0;
      for (int i = 0; i < 32; ++i)
        if (fabs(y[i]) > amax) amax = fabs(y[i]);
      uint8_t sb = scale_byte_of(amax, sr);
      s[r * nb + b] = sb;
      double scale = ldexp(1.0, (int)sb - 127);
      for (int i = 0; i < 32; i += 2) {
        uint8_t c[2];
        for (int h = 0; h < 2; ++h) {
          double v = fabs(y[i + h]) / scale; /* exact: a power-of-two scale */
          uint8_t code;
          if (sr)
            code = oracle_sr_code(v, oracle_sr_uniform16(seed, (uint64_t)(r * K + b * 32 + i + h)));
          else
            code = e2m1_magnitude_code(v);
          if (neg[i + h]) code |= 8;
          c[h] = code;
        }
        q[r * (K / 2) + (b * 32 + i) / 2] = (uint8_t)(c[0] | (c[1] << 4));
      }
    }
  }
  return bad;
}

typedef struct {
  const uint16_t* w;
  int64_t r0, r1, K;
  uint32_t flags;
  const uint32_t* signs;
  uint64_t seed;
  uint8_t *q, *s;
  int64_t bad;
} quant_ex_job;

static void* quant_ex_run(void* arg) {
  quant_ex_job* j = (quant_ex_job*)arg;
  j->bad = quantize_ex_rows(j->w, j->r0, j->r1, j->K, j->flags, j->signs, j->seed, j->q, j->s);
  return NULL;
}

/* bf16 [rows][K] -> codes + scale bytes with the optional transform and
 * stochastic rounding above; rows split over threads.  Returns the number of
 * blocks holding a NaN or infinity. */
int64_t oracle_mxfp4_quantize_sr_rht(const uint16_t* w, int64_t rows, int64_t K, uint32_t flags,
                                     const uint32_t* signs, uint64_t seed, uint8_t* q, uint8_t* s,
                                     int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (rows < 64) nthreads = 1;
  pthread_t th[256];
  quant_ex_job jobs[256];
  int created[256];
  int64_t chunk = (rows + nthreads - 1) / nthreads;
  int used = 0;
  for (int t = 0; t < nthreads; ++t) {
    quant_ex_job j = {w, t * chunk, (t + 1) * chunk < rows ? (t + 1) * chunk : rows, K, flags,
                      signs, seed, q, s, 0};
    jobs[t] = j;
    if (jobs[t].r0 >= jobs[t].r1) break;
    created[t] = pthread_create(&th[t], NULL, quant_ex_run, &jobs[t]) == 0;
    if (!created[t]) quant_ex_run(&jobs[t]);
    used = t + 1;
  }
  int64_t bad = 0;
  for (int t = 0; t < used; ++t) {
    if (created[t]) pthread_join(th[t], NULL);
    bad += jobs[t].bad;
  }
  return bad;
}

/* ------------------------------------------------------------------ routing */

/* token-choice top-k with softmax over the selected logits [P2 s4, P3] */
void oracle_route(const float* logits, int64_t T, int E, int k, int32_t* idx, double* w) {
  for (int64_t t = 0; t < T; ++t) {
    const float* l = logits + t * E;
    unsigned char taken[256];
    memset(taken, 0, sizeof taken);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        /* strict '>' keeps the lowest index among equal logits; -0 == +0 */
        if (best < 0 || l[e] > l[best]) best = e;
      }
      taken[best] = 1;
      idx[t * k + j] = best;
    }
    double lmax = (double)l[idx[t * k]];
    double z = 0.0;
    for (int j = 0; j < k; ++j) z += exp((double)l[idx[t * k + j]] - lmax);
    for (int j = 0; j < k; ++j) w[t * k + j] = exp((double)l[idx[t * k + j]] - lmax) / z;
  }
}

/* router scores [P2 s4: a router scores every token against every expert]:
 * logits[t][e] = sum_d x[t][d] * w[e][d] over bf16 inputs, in fp64, d ascending */
void oracle_router_logits(const uint16_t* x, const uint16_t* w, int64_t T, int D, int E,
                          double* logits) {
  for (int64_t t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int d = 0; d < D; ++d)
        acc += oracle_bf16_value(x[t * D + d]) * oracle_bf16_value(w[(int64_t)e * D + d]);
      logits[t * E + e] = acc;
    }
}

/* group slots by expert: counting sort, ascending slot order within expert */
void oracle_permute(const int32_t* idx, int64_t T, int E, int k, int32_t* counts,
                    int32_t* offsets, int32_t* sorted_slot, int32_t* slot_pos) {
  const int64_t S = T * k;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t s = 0; s < S; ++s) counts[idx[s]]++;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* fill = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
  for (int e = 0; e < E; ++e) fill[e] = offsets[e];
  for (int64_t s = 0; s < S; ++s) {
    int32_t p = fill[idx[s]]++;
    sorted_slot[p] = (int32_t)s;
    slot_pos[s] = p;
  }
  free(fill);
}

/* x_perm[p] = x[sorted_slot[p] / k] */
void oracle_gather(const uint16_t* x, const int32_t* sorted_slot, int64_t S, int k, int D,
                   uint16_t* x_perm) {
  for (int64_t p = 0; p < S; ++p)
    memcpy(x_perm + p * D, x + (int64_t)(sorted_slot[p] / k) * D, sizeof(uint16_t) * D);
}

/* ---------------------------------------------------------------- expert MLP */

/* one expert applied to one bf16 row: SwiGLU MLP [P2 s4] with weights already
 * decoded to double [P3 "Hardware optimisation"].
 *   wgu: [2F][D] (gate rows first), wdn: [D][F]
 *   h_out [F], y_out [D] as bf16 bit patterns */
static void expert_row(const uint16_t* xrow, int D, int F, const double* wgu, const double* wdn,
                       uint16_t* h_out, uint16_t* y_out, double* hbuf) {
  for (int n = 0; n < F; ++n) {
    const double* wg = wgu + (int64_t)n * D;
    const double* wu = wgu + (int64_t)(F + n) * D;
    double g = 0.0, u = 0.0;
    for (int d = 0; d < D; ++d) {
      double xv = oracle_bf16_value(xrow[d]);
      g += xv * wg[d];
      u += xv * wu[d];
    }
    double silu = g / (1.0 + exp(-g));
    uint16_t hb = oracle_bf16_round(silu * u);
    if (h_out) h_out[n] = hb;
    hbuf[n] = oracle_bf16_value(hb);
  }
  for (int d = 0; d < D; ++d) {
    const double* wd = wdn + (int64_t)d * F;
    double acc = 0.0;
    for (int n = 0; n < F; ++n) acc += hbuf[n] * wd[n];
    y_out[d] = oracle_bf16_round(acc);
  }
}

typedef struct {
  const uint16_t* rows; /* [n][D] */
  int64_t n;
  int D, F;
  const double* wgu;
  const double* wdn;
  uint16_t* h; /* [n][F] or NULL */
  uint16_t* y; /* [n][D] */
  int64_t lo, hi;
} mlp_job;

static void* mlp_run(void* arg) {
  mlp_job* j = (mlp_job*)arg;
  double* hbuf = (double*)malloc(sizeof(double) * (size_t)j->F);
  for (int64_t r = j->lo; r < j->hi; ++r)
    expert_row(j->rows + r * j->D, j->D, j->F, j->wgu, j->wdn,
               j->h ? j->h + r * j->F : NULL, j->y + r * j->D, hbuf);
  free(hbuf);
  return NULL;
}

/* apply one expert (decoded weights) to n rows, split over nthreads */
static void expert_rows_parallel(const uint16_t* rows, int64_t n, int D, int F,
                                 const double* wgu, const double* wdn, uint16_t* h, uint16_t* y,
                                 int nthreads) {
  if (n <= 0) return;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (nthreads > n) nthreads = (int)n;
  pthread_t th[256];
  mlp_job jobs[256];
  int created[256];
  int64_t chunk = (n + nthreads - 1) / nthreads;
  int used = 0;
  for (int t = 0; t < nthreads; ++t) {
    mlp_job j = {rows, n, D, F, wgu, wdn, h, y, t * chunk, (t + 1) * chunk < n ? (t + 1) * chunk : n};
    jobs[t] = j;
    if (jobs[t].lo >= jobs[t].hi) break;
    created[t] = pthread_create(&th[t], NULL, mlp_run, &jobs[t]) == 0;
    if (!created[t]) mlp_run(&jobs[t]);
    used = t + 1;
  }
  for (int t = 0; t < used; ++t)
    if (created[t]) pthread_join(th[t], NULL);
}

/* decode one expert's gate/up [2F][D] and down [D][F] matrices to double */
static int decode_expert(int e, int D, int F, const uint8_t* wgu_q, const uint8_t* wgu_s,
                         const uint8_t* wdn_q, const uint8_t* wdn_s, double* wgu, double* wdn) {
  const int64_t gu_rows = 2 * (int64_t)F;
  oracle_mxfp4_decode(wgu_q + (int64_t)e * gu_rows * (D / 2), wgu_s + (int64_t)e * gu_rows * (D / 32),
                      gu_rows, D, wgu);
  oracle_mxfp4_decode(wdn_q + (int64_t)e * D * (F / 2), wdn_s + (int64_t)e * D * (F / 32), D, F, wdn);
  return 0;
}

/* grouped expert MLP over permuted rows: rows [offsets[e], offsets[e+1])
 * belong to expert e */
int oracle_expert_mlp(const uint16_t* x_perm, const int32_t* offsets, int E, int D, int F,
                      const uint8_t* wgu_q, const uint8_t* wgu_s, const uint8_t* wdn_q,
                      const uint8_t* wdn_s, uint16_t* h, uint16_t* y, int nthreads) {
  double* wgu = (double*)malloc(sizeof(double) * 2 * (size_t)F * D);
  double* wdn = (double*)malloc(sizeof(double) * (size_t)D * F);
  if (!wgu || !wdn) {
    free(wgu);
    free(wdn);
    return -1;
  }
  for (int e = 0; e < E; ++e) {
    int64_t r0 = offsets[e], r1 = offsets[e + 1];
    if (r1 <= r0) continue;
    decode_expert(e, D, F, wgu_q, wgu_s, wdn_q, wdn_s, wgu, wdn);
    expert_rows_parallel(x_perm + r0 * D, r1 - r0, D, F, wgu, wdn, h ? h + r0 * F : NULL,
                         y + r0 * D, nthreads);
  }
  free(wgu);
  free(wdn);
  return 0;
}

/* The same grouped expert MLP with unquantised bf16 weights, the comparison
 * point the pages set against MXFP4 (the bf16 path takes about 4x the
 * memory: "Tricks from OpenAI gpt-oss ...", section 7; agentlenshq (ja),
 * "What is MXFP4").  Weights: wgu [E][2F][D], wdn [E][D][F] as bf16 bit
 * patterns; every step as in oracle_expert_mlp, the weights taken at their
 * exact bf16 values instead of decoded codes. */
int oracle_expert_mlp_bf16(const uint16_t* x_perm, const int32_t* offsets, int E, int D, int F,
                           const uint16_t* wgu_bf16, const uint16_t* wdn_bf16, uint16_t* h,
                           uint16_t* y, int nthreads) {
  double* wgu = (double*)malloc(sizeof(double) * 2 * (size_t)F * D);
  double* wdn = (double*)malloc(sizeof(double) * (size_t)D * F);
  if (!wgu || !wdn) {
    free(wgu);
    free(wdn);
    return -1;
  }
  for (int e = 0; e < E; ++e) {
    int64_t r0 = offsets[e], r1 = offsets[e + 1];
    if (r1 <= r0) continue;
    const uint16_t* gsrc = wgu_bf16 + (int64_t)e * 2 * F * D;
    const uint16_t* dsrc = wdn_bf16 + (int64_t)e * D * F;
    for (int64_t i = 0; i < 2 * (int64_t)F * D; ++i) wgu[i] = oracle_bf16_value(gsrc[i]);
    for (int64_t i = 0; i < (int64_t)D * F; ++i) wdn[i] = oracle_bf16_value(dsrc[i]);
    expert_rows_parallel(x_perm + r0 * D, r1 - r0, D, F, wgu, wdn, h ? h + r0 * F : NULL,
                         y + r0 * D, nthreads);
  }
  free(wgu);
  free(wdn);
  return 0;
}

/* out[t][d] = bf16( sum_j w[t][j] * y_perm[slot_pos[t*k+j]][d] ), j ascending */
void oracle_combine(const uint16_t* y_perm, const int32_t* slot_pos, const double* w, int64_t T,
                    int k, int D, uint16_t* out) {
  for (int64_t t = 0; t < T; ++t)
    for (int d = 0; d < D; ++d) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j)
        acc += w[t * k + j] * oracle_bf16_value(y_perm[(int64_t)slot_pos[t * k + j] * D + d]);
      out[t * D + d] = oracle_bf16_round(acc);
    }
}

/* the whole layer in the library's step order: route, permute, gather,
 * grouped expert MLP, combine */
int oracle_layer_forward(const uint16_t* x, const float* logits, int64_t T, int E, int k, int D,
                         int F, const uint8_t* wgu_q, const uint8_t* wgu_s, const uint8_t* wdn_q,
                         const uint8_t* wdn_s, uint16_t* out, int nthreads) {
  const int64_t S = T * k;
  int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(S > 0 ? S : 1));
  double* w = (double*)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1));
  int32_t* counts = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  int32_t* offsets = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
  int32_t* sorted_slot = (int32_t*)malloc(sizeof(int32_t) * (size_t)(S > 0 ? S : 1));
  int32_t* slot_pos = (int32_t*)malloc(sizeof(int32_t) * (size_t)(S > 0 ? S : 1));
  uint16_t* x_perm = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(S > 0 ? S : 1) * D);
  uint16_t* y = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(S > 0 ? S : 1) * D);
  int rc = -1;
  if (idx && w && counts && offsets && sorted_slot && slot_pos && x_perm && y) {
    oracle_route(logits, T, E, k, idx, w);
    oracle_permute(idx, T, E, k, counts, offsets, sorted_slot, slot_pos);
    oracle_gather(x, sorted_slot, S, k, D, x_perm);
    rc = oracle_expert_mlp(x_perm, offsets, E, D, F, wgu_q, wgu_s, wdn_q, wdn_s, NULL, y,
                           nthreads);
    if (rc == 0) oracle_combine(y, slot_pos, w, T, k, D, out);
  }
  free(idx);
  free(w);
  free(counts);
  free(offsets);
  free(sorted_slot);
  free(slot_pos);
  free(x_perm);
  free(y);
  return rc;
}

/* the layer for selected tokens only, written per token with no permutation:
 * for token t, route it, run each chosen expert on x[t], mix with the
 * softmax weights.  out_rows[i] is the output row of token tokens[i];
 * y_rows (nullable) receives the bf16 expert outputs [i][j][D]. */
int oracle_layer_tokens(const uint16_t* x, const float* logits, int E, int k, int D, int F,
                        const uint8_t* wgu_q, const uint8_t* wgu_s, const uint8_t* wdn_q,
                        const uint8_t* wdn_s, const int64_t* tokens, int64_t n_tokens,
                        uint16_t* out_rows, uint16_t* y_rows, int nthreads) {
  int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n_tokens * k + 1));
  double* w = (double*)malloc(sizeof(double) * (size_t)(n_tokens * k + 1));
  uint16_t* y = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(n_tokens * k + 1) * D);
  double* wgu = (double*)malloc(sizeof(double) * 2 * (size_t)F * D);
  double* wdn = (double*)malloc(sizeof(double) * (size_t)D * F);
  uint16_t* row = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(n_tokens + 1) * D);
  int rc = -1;
  if (idx && w && y && wgu && wdn && row) {
    for (int64_t i = 0; i < n_tokens; ++i)
      oracle_route(logits + tokens[i] * E, 1, E, k, idx + i * k, w + i * k);
    /* each needed expert is decoded once; its rows are computed in token order */
    for (int e = 0; e < E; ++e) {
      int64_t n = 0;
      for (int64_t i = 0; i < n_tokens; ++i)
        for (int j = 0; j < k; ++j)
          if (idx[i * k + j] == e) memcpy(row + (n++) * D, x + tokens[i] * D, sizeof(uint16_t) * D);
      if (n == 0) continue;
      decode_expert(e, D, F, wgu_q, wgu_s, wdn_q, wdn_s, wgu, wdn);
      uint16_t* yr = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)n * D);
      expert_rows_parallel(row, n, D, F, wgu, wdn, NULL, yr, nthreads);
      int64_t m = 0;
      for (int64_t i = 0; i < n_tokens; ++i)
        for (int j = 0; j < k; ++j)
          if (idx[i * k + j] == e) memcpy(y + (i * k + j) * D, yr + (m++) * D, sizeof(uint16_t) * D);
      free(yr);
    }
    for (int64_t i = 0; i < n_tokens; ++i)
      for (int d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int j = 0; j < k; ++j) acc += w[i * k + j] * oracle_bf16_value(y[(i * k + j) * D + d]);
        out_rows[i * D + d] = oracle_bf16_round(acc);
      }
    /* optional: the k expert outputs of each token, [n_tokens][k][D] */
    if (y_rows) memcpy(y_rows, y, sizeof(uint16_t) * (size_t)(n_tokens * k) * D);
    rc = 0;
  }
  free(idx);
  free(w);
  free(y);
  free(wgu);
  free(wdn);
  free(row);
  return rc;
}
