// Training-style bf16 -> MXFP4 quantiser: optional random-sign Hadamard
// transform of every 32-element block and optional stochastic rounding.
//
// "MXFP4-based MoE technical review", sections 2 and 4, names stochastic
// rounding and a random Hadamard transform as what keeps MXFP4 training close
// to bf16.  What this kernel computes, per 32-element block of a row:
//   * transform (flag MOE_QUANT_RHT): y = H (s . x), H the unnormalised 32-point
//     Sylvester Hadamard matrix (H[i][j] = (-1)^popcount(i & j)), s the signs
//     of the block's column given by the caller.  H diag(s) times its
//     transpose is 32 I, so a GEMM whose two operands carry the same transform
//     along K returns 32 times the plain product.  y is exact: the butterfly
//     runs in fp64, where sums of 32 bf16 terms whose exponents span less than
//     40 binades carry no rounding;
//   * scale byte: floor(log2 amax) - 2 + 127, as in the deterministic
//     quantiser, or, with stochastic rounding, the smallest exponent that keeps
//     amax / scale <= 6 (one more when the significand of amax is above 1.5),
//     so that no element clips and the rounding stays unbiased; clamped to
//     [0, 254];
//   * codes: |y| / scale (exact) rounded to nearest even onto
//     {0, .5, 1, 1.5, 2, 3, 4, 6}, or (flag MOE_QUANT_SR) to the upper grid
//     neighbour when u / 2^16 < (v - lo) / (hi - lo), u the element's 16-bit
//     uniform from Philox4x32-10 (Salmon, Moraes, Dror and Shaw, SC 2011):
//     element n of the call uses counter (n / 8, 0, 0) under the 64-bit seed,
//     output word (n % 8) / 2, low half for even n;
//   * sign bit: y < 0 with the transform (an exact zero is +0), else the sign
//     bit of x.  With no flag the call is mxfp4_quantize itself.
//
// Layout: one thread per 32-element block.  A warp loads 32 consecutive blocks
// (2 KB) with coalesced 16-byte loads into a padded shared-memory stage (a
// block's 64 bytes take 80, so the per-thread reads are free of bank
// conflicts), widens its own block to 32 doubles, transforms, encodes and
// writes its 16 code bytes (the warp's 512 are contiguous) and its scale byte.
// The fp64 butterfly, Philox and the integer encoding make the kernel
// instruction-bound rather than HBM-bound.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStageStride = 5;  // uint4 slots per block in the stage (4 + 1 pad)

constexpr uint32_t kPhiloxM0 = 0xD2511F53u, kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u, kPhiloxW1 = 0xBB67AE85u;

// Philox4x32-10 of counter c under key (k0, k1)
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t lo0 = kPhiloxM0 * c.x, hi0 = __umulhi(kPhiloxM0, c.x);
    const uint32_t lo1 = kPhiloxM1 * c.z, hi1 = __umulhi(kPhiloxM1, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += kPhiloxW0;
    k1 += kPhiloxW1;
  }
  return c;
}

constexpr double kTwo52 = 4503599627370496.0;  // 2^52: adding it leaves an integer in the low word
constexpr double kTwo36 = 68719476736.0;       // 2^36: the low word then counts steps of 2^-16

// E2M1 magnitude code of v = |y| / scale >= 0 (exact), without branches.
// The code grid {0, .5, 1, 1.5, 2, 3, 4, 6} has step g = 0.5 below 2 and
// g = 2^(e-1) in the binade [2^e, 2^(e+1)), e >= 1.  With e = max(floor(log2
// v), 0) (from the high word of max(v, 1)), a = v / g is exact and lies in
// [0, 2) below 1 and in [2, 4) above; the grid point below v is then n =
// floor(a) steps, and the code is 2 e + n, plus one when rounded up, capped
// at 7 (6.0; only a scale clamped at 254 reaches it).  Code parity equals n's
// parity, so ties to even on the integer grid of a are ties to an even code.
//   nearest:    adding 2^52 in round-to-nearest-even leaves n + up in the low word;
//   stochastic: adding it rounding toward zero leaves n; up when
//               n + u / 2^16 < a, i.e. u / 2^16 < (v - lo) / (hi - lo), with
//               n + u / 2^16 built exactly as 2^36 + (n 2^16 + u) 2^-16 - 2^36.
// rw holds the element's uniform in its low (half 0) or high (half 1) 16 bits.
template <bool SR>
__device__ __forceinline__ uint32_t e2m1_code(double v, uint32_t rw, int half) {
  const int th = max(__double2hiint(v), 0x3FF00000);                         // max(v, 1)
  const double inv_g = __hiloint2double(0x7FF00000 - (th & 0x7FF00000), 0);  // 2^(1 - e)
  const double a = v * inv_g;
  uint32_t c;
  if (SR) {
    const uint32_t n = static_cast<uint32_t>(__double2loint(__dadd_rz(a, kTwo52)));
    const uint32_t lo = __byte_perm(rw, n, half ? 0x5432 : 0x5410);  // n 2^16 + u
    const double nu = __hiloint2double(0x42300000, static_cast<int>(lo)) - kTwo36;
    c = n + (nu < a ? 1u : 0u);
  } else {
    c = static_cast<uint32_t>(__double2loint(__dadd_rn(a, kTwo52)));
  }
  c += 2u * static_cast<uint32_t>((th >> 20) - 1023);
  return min(c, 7u);
}

template <bool RHT, bool SR>
__global__ void __launch_bounds__(kThreads) quantize_sr_rht_kernel(
    const uint4* __restrict__ w, int64_t nblocks, int64_t nbk, int64_t stride_mod,
    const uint32_t* __restrict__ signs, uint32_t key0, uint32_t key1, uint4* __restrict__ q,
    uint8_t* __restrict__ s, int32_t* __restrict__ status) {
  __shared__ uint4 stage[kWarps][32 * kStageStride];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t warp0 = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  int64_t col = (warp0 * 32 + lane) % nbk;  // block column of this lane's block
  for (int64_t base = warp0 * 32; base < nblocks; base += nwarps * 32) {
    // coalesced 16-byte loads of the warp's 32 blocks into the stage
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int p = lane + 32 * j;  // piece p of the warp: block p / 4, quarter p % 4
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (base * 4 + p < nblocks * 4) v = __ldg(w + base * 4 + p);
      stage[warp][(p >> 2) * kStageStride + (p & 3)] = v;
    }
    __syncwarp();
    uint32_t word[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 v = stage[warp][lane * kStageStride + j];
      word[4 * j] = v.x;
      word[4 * j + 1] = v.y;
      word[4 * j + 2] = v.z;
      word[4 * j + 3] = v.w;
    }
    __syncwarp();
    const int64_t blk = base + lane;
    const bool valid = blk < nblocks;
    const uint32_t sgn = (RHT && valid) ? __ldg(signs + col) : 0u;

    // bf16 -> fp32 bit pattern (a shift), the sign flip of the transform on
    // its sign bit, then the exact widening to fp64 (subnormals included;
    // Inf and NaN stay non-finite and are caught through the block maximum)
    double y[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const uint32_t wd = word[t >> 1];
      uint32_t f = (t & 1) ? (wd & 0xFFFF0000u) : (wd << 16);
      if (RHT) f ^= (sgn << (31 - t)) & 0x80000000u;
      y[t] = static_cast<double>(__uint_as_float(f));
    }
    if (RHT) {
      // in-place fast Walsh-Hadamard transform, natural (Sylvester) order
#pragma unroll
      for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if ((i & h) == 0) {
            const double a = y[i], c = y[i + h];
            y[i] = a + c;
            y[i + h] = a - c;
          }
        }
      }
    }

    // block maximum of |y| (exact), and the non-finite test: with the
    // transform y[0] is the signed sum of the whole block, so any Inf or NaN
    // input leaves it non-finite; without it, the plain sum of the block
    double amax = 0.0, total = 0.0;
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      amax = fmax(amax, fabs(y[t]));
      if (!RHT) total += y[t];
    }
    if (RHT) total = y[0];
    const bool nonfinite = (static_cast<uint32_t>(__double2hiint(total)) & 0x7FF00000u) == 0x7FF00000u;
    const uint32_t amax_hi = static_cast<uint32_t>(__double2hiint(amax));
    int sb = 0;
    if (amax_hi != 0) {
      // floor(log2 amax) - 2 + 127; with stochastic rounding one more when
      // the significand of amax is above 1.5
      sb = static_cast<int>(amax_hi >> 20) - 1023 + 125;
      if (SR) {
        const uint32_t frac_hi = amax_hi & 0xFFFFFu;
        sb += (frac_hi > 0x80000u || (frac_hi == 0x80000u && __double2loint(amax) != 0)) ? 1 : 0;
      }
      sb = min(max(sb, 0), 254);
    }
    const double inv_scale = __hiloint2double((127 - sb + 1023) << 20, 0);  // 2^(127 - sb)

    uint32_t out[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint4 rnd = make_uint4(0u, 0u, 0u, 0u);
      if (SR) {
        const uint64_t ctr = static_cast<uint64_t>(blk) * 4 + g;  // (32 blk + 8 g) / 8
        rnd = philox4x32_10(make_uint4(static_cast<uint32_t>(ctr), static_cast<uint32_t>(ctr >> 32),
                                       0u, 0u),
                            key0, key1);
      }
      const uint32_t rw[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
      uint32_t o = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int t = 8 * g + e;
        uint32_t c = e2m1_code<SR>(fabs(y[t]) * inv_scale, rw[e >> 1], e & 1);
        // sign bit: that of x without the transform (-0 included); with it,
        // y < 0 only (an exact zero is +0)
        if (RHT)
          c |= y[t] < 0.0 ? 8u : 0u;
        else
          c |= (static_cast<uint32_t>(__double2hiint(y[t])) >> 28) & 8u;
        o |= c << (4 * e);
      }
      out[g] = o;
    }
    if (valid) {
      q[blk] = make_uint4(out[0], out[1], out[2], out[3]);
      s[blk] = static_cast<uint8_t>(sb);
      if (nonfinite) record_status(status, MOE_ERR_NONFINITE);
    }
    col += stride_mod;
    if (col >= nbk) col -= nbk;
  }
}

using KernelFn = void (*)(const uint4*, int64_t, int64_t, int64_t, const uint32_t*, uint32_t,
                          uint32_t, uint4*, uint8_t*, int32_t*);

KernelFn pick(uint32_t flags) {
  switch (flags) {
    case MOE_QUANT_RHT: return quantize_sr_rht_kernel<true, false>;
    case MOE_QUANT_SR: return quantize_sr_rht_kernel<false, true>;
    default: return quantize_sr_rht_kernel<true, true>;
  }
}

}  // namespace
}  // namespace moe

extern "C" moe_status mxfp4_quantize_sr_rht(const uint16_t* w_bf16, int64_t rows, int64_t K,
                                            uint32_t flags, const uint32_t* rht_signs,
                                            uint64_t seed, uint8_t* q_packed, uint8_t* scales,
                                            int32_t* d_status, moe_stream stream) {
  using namespace moe;
  if (flags & ~static_cast<uint32_t>(MOE_QUANT_RHT | MOE_QUANT_SR)) return MOE_ERR_INVALID_ARG;
  // no flag: the deterministic quantiser's bytes, from its own kernel
  if (flags == 0) return mxfp4_quantize(w_bf16, rows, K, q_packed, scales, d_status, stream);
  if (rows < 0 || K < 32 || (K % 32) != 0) return MOE_ERR_SHAPE;
  if (rows > 0 && K > (int64_t(1) << 40) / rows) return MOE_ERR_SHAPE;
  if (rows == 0) return MOE_OK;
  if (!w_bf16 || !q_packed || !scales) return MOE_ERR_INVALID_ARG;
  if ((flags & MOE_QUANT_RHT) && !rht_signs) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w_bf16) || !aligned16(q_packed) || !aligned16(scales)) return MOE_ERR_INVALID_ARG;
  if (rht_signs && (reinterpret_cast<uintptr_t>(rht_signs) & 3u)) return MOE_ERR_INVALID_ARG;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_device();
  if (st != MOE_OK) return st;
  const int64_t nblocks = rows * (K / 32);
  const int64_t nbk = K / 32;
  const int64_t want = (nblocks + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const int grid = static_cast<int>(want < cap ? want : cap);
  const int64_t stride_mod = (static_cast<int64_t>(grid) * kThreads) % nbk;
  pick(flags)<<<grid, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint4*>(w_bf16), nblocks, nbk, stride_mod, rht_signs,
      static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32),
      reinterpret_cast<uint4*>(q_packed), scales, d_status);
  return launch_status();
}
