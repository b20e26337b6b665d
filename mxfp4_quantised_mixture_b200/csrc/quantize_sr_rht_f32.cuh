// One 32-element block of the training-style quantiser in fp32, for the
// blocks where fp32 holds the transformed values exactly.
//
// "MXFP4-based MoE technical review", sections 2 and 4: stochastic rounding
// and a random Hadamard transform.  The arithmetic is that of the fp64 path in
// quantize_sr_rht.cu (same scale rule, same rounding decisions, same bits);
// fp32 only serves the blocks where every value it forms is exact:
//   * without the transform y = x, and every finite bf16 value is an fp32
//     value;
//   * with it, each y (and each partial sum of the butterfly) is a signed sum
//     of up to 32 of the block's bf16 values.  With ee = max(exponent field,
//     1) of a nonzero input (a subnormal bf16 has the spacing of field 1),
//     every input is a multiple of 2^(ee_min - 134) and every sum is below
//     2^(ee_max - 121) in magnitude, so a sum holds at most
//     ee_max - ee_min + 13 significant bits: exact in fp32's 24 whenever
//     ee_max - ee_min <= 11, and with ee_max <= 247 nothing overflows.
//     Normal weights span far fewer binades within a block, so nearly every
//     block takes this path; the rest take the fp64 one.
// Once y is exact, v = |y| / scale is too (a power-of-two scale, v well
// inside fp32's range), and the rounding decisions below read v's fp32 bit
// fields exactly as the fp64 path reads its fp64 fields.
#pragma once

#include <stdint.h>
#include <string.h>

#if defined(__CUDACC__)
#define MOE_HD __host__ __device__ __forceinline__
#else
#define MOE_HD inline
#endif

namespace moe {
namespace srq {

MOE_HD float bits_f32(uint32_t u) {
#if defined(__CUDA_ARCH__)
  return __uint_as_float(u);
#else
  float f;
  memcpy(&f, &u, 4);
  return f;
#endif
}

MOE_HD uint32_t f32_bits(float f) {
#if defined(__CUDA_ARCH__)
  return __float_as_uint(f);
#else
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
#endif
}

// Whether fp32 holds the block exactly (see above).  xf: the 32 inputs as
// fp32 bit patterns (bf16 bits << 16, the transform's sign flips applied).
template <bool RHT>
MOE_HD bool block_fits_f32(const uint32_t (&xf)[32]) {
  uint32_t emax = 0, emin = 255;
#pragma unroll
  for (int t = 0; t < 32; ++t) {
    const uint32_t mag = xf[t] & 0x7FFFFFFFu;
    const uint32_t e = mag >> 23;
    const uint32_t ee = e > 1u ? e : 1u;
    if (mag != 0u) {
      emax = ee > emax ? ee : emax;
      emin = ee < emin ? ee : emin;
    }
  }
  if (!RHT) return emax < 255u;                        // finite: y = x
  return emax == 0u || (emax <= 247u && emax - emin <= 11u);  // all zero, or exact sums
}

// E2M1 magnitude code of v = |y| / scale >= 0 from v's fp32 bit fields:
//   v >= 1:       binade e holds 2^e and 1.5 2^e: base code 2 + 2e + (top
//                 mantissa bit); the other 22 mantissa bits are the fraction
//                 of the gap (2^(e-1)) to the next code; saturates at 7;
//   v in [.5, 1): base 1 (0.5); the 23 mantissa bits are the fraction of 0.5;
//   v < .5:       base 0; fraction 2 v.
// Round to nearest even, or, with stochastic rounding, up when the 16-bit
// uniform u / 2^16 is below the fraction.
template <bool SR>
MOE_HD uint32_t e2m1_code_f32(float v, uint32_t u) {
  const uint32_t vb = f32_bits(v);
  const uint32_t ev = vb >> 23;  // v >= 0: no sign bit
  uint32_t code;
  if (ev >= 127u) {
    const uint32_t base = 2u + 2u * (ev - 127u) + ((vb >> 22) & 1u);
    const uint32_t R = vb & 0x3FFFFFu;  // 22 bits
    bool up;
    if (SR)
      up = (u << 6) < R;
    else
      up = R > 0x200000u || (R == 0x200000u && (base & 1u));
    code = base + (up ? 1u : 0u);
    code = code < 7u ? code : 7u;
  } else if (ev == 126u) {
    const uint32_t R = vb & 0x7FFFFFu;  // 23 bits
    const bool up = SR ? (u << 7) < R : R >= 0x400000u;
    code = up ? 2u : 1u;
  } else {
    const bool up = SR ? static_cast<float>(u) < v * 131072.0f : v > 0.25f;
    code = up ? 1u : 0u;
  }
  return code;
}

// One block: xf as for block_fits_f32 (which must hold); words(g) returns
// the four uniform words of element group g (element 8 g + e takes half
// e & 1 of word e >> 1; only called with stochastic rounding).  Outputs: the
// 16 code bytes as four words (element 8 g + e in nibble e of out[g]), the
// scale byte, and whether the block holds Inf/NaN.
template <bool RHT, bool SR, typename Words>
MOE_HD void encode_block_f32(const uint32_t (&xf)[32], const Words& words, uint32_t (&out)[4],
                             int& sb_out, bool& nonfinite) {
  float y[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) y[t] = bits_f32(xf[t]);
  if (RHT) {
    // in-place fast Walsh-Hadamard transform, natural (Sylvester) order
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if ((i & h) == 0) {
          const float a = y[i], c = y[i + h];
          y[i] = a + c;
          y[i + h] = a - c;
        }
      }
    }
  }
  uint32_t amax = 0;
#pragma unroll
  for (int t = 0; t < 32; ++t) {
    const uint32_t m = f32_bits(y[t]) & 0x7FFFFFFFu;
    amax = m > amax ? m : amax;
  }
  nonfinite = amax >= 0x7F800000u;
  // floor(log2 amax) - 2 + 127, one more under stochastic rounding when the
  // significand is above 1.5; a subnormal or zero maximum gives 0
  int sb = 0;
  if (amax >= 0x00800000u) {
    sb = static_cast<int>(amax >> 23) - 127 + 125;
    if (SR && (amax & 0x7FFFFFu) > 0x400000u) ++sb;
    sb = sb < 0 ? 0 : (sb > 254 ? 254 : sb);
  }
  const float inv_scale = bits_f32(static_cast<uint32_t>(127 - sb + 127) << 23);  // 2^(127 - sb)
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint32_t rw[4] = {0u, 0u, 0u, 0u};
    if (SR) words(g, rw);
    uint32_t o = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int t = 8 * g + e;
      const uint32_t u = (rw[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
      const uint32_t yb = f32_bits(y[t]);
      uint32_t c = e2m1_code_f32<SR>(bits_f32(yb & 0x7FFFFFFFu) * inv_scale, u);
      // sign bit: that of x without the transform (-0 included); with it,
      // y < 0 only (an exact zero of the butterfly is +0)
      c |= (RHT ? (yb > 0x80000000u ? 1u : 0u) : (yb >> 31)) << 3;
      o |= c << (4 * e);
    }
    out[g] = o;
  }
  sb_out = sb;
}

}  // namespace srq
}  // namespace moe
