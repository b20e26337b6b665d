// bf16 -> MXFP4 block quantiser.
//
// MXFP4 (E2M1 elements, one shared power-of-two scale per 32 elements):
// "Tricks from OpenAI gpt-oss you can use with transformers" (summary),
// section 6; agentlenshq "Transformers ... GPT-OSS" (ja), "What is MXFP4";
// the scale is the OCP MX E8M0 byte ("MXFP4-based MoE technical review",
// section 1), exponent floor(log2 amax) - 2 so that the block maximum lands in
// the top binade [4, 8) of E2M1.
//
// Layout: the input is a flat sequence of 32-element blocks (rows of K with
// K % 32 == 0).  Four consecutive lanes own one block, 8 elements (16 bytes)
// each: a warp reads 512 contiguous bytes and writes 128 contiguous code
// bytes plus 8 contiguous scale bytes per step, and each lane keeps
// kUnroll = 4 such 16-byte loads in flight.  The element codes come from
// sm_100's E2M1 conversion (cvt.rn.satfinite.e2m1x2.f32: round to nearest,
// ties to even, saturating at 6, sign kept), applied to v = x / scale in fp32.
// v is below 8, and exact wherever it could reach a nonzero code (a bf16
// value times a power of two is a normal fp32 number down to 2^-126); smaller
// v may underflow, keeping its sign, and gives code 0 or 8 either way.  With
// two elements per conversion, one max per element pair and one multiply per
// element the kernel is a stream bound by HBM (2 bytes read, 17/32 byte
// written per element).
#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

// E2M1 codes of 8 fp32 values (element 0 in the low nibble of the result)
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&f)[8]) {
  uint32_t out;
  asm("{\n"
      ".reg .b8 c0, c1, c2, c3;\n"
      "cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n"
      "cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n"
      "cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n"
      "cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n"
      "mov.b32 %0, {c0, c1, c2, c3};\n"
      "}"
      : "=r"(out)
      : "f"(f[0]), "f"(f[1]), "f"(f[2]), "f"(f[3]), "f"(f[4]), "f"(f[5]), "f"(f[6]), "f"(f[7]));
  return out;
}

__device__ __forceinline__ uint32_t encode8(uint4 v, float inv_scale) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float f[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // x / scale: a bf16 value times a power of two (exact unless it underflows)
    f[2 * j] = __uint_as_float(w[j] << 16) * inv_scale;
    f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u) * inv_scale;
  }
  return cvt_e2m1x8(f);
}

// largest bf16 magnitude pattern of 8 elements (orders like the values for
// finite bf16; >= 0x7F80 exactly when one of them is Inf or NaN)
__device__ __forceinline__ uint32_t max_magnitude8(uint4 v) {
  const uint32_t m = 0x7FFF7FFFu;
  const uint32_t a = __vmaxu2(__vmaxu2(v.x & m, v.y & m), __vmaxu2(v.z & m, v.w & m));
  return max(a & 0xFFFFu, a >> 16);
}

__global__ void __launch_bounds__(kThreads) quantize_kernel(const uint4* __restrict__ w,
                                                           int64_t nquarters,
                                                           uint32_t* __restrict__ q,
                                                           uint8_t* __restrict__ s,
                                                           int32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  for (int64_t base = warp0 * 32 * kUnroll; base < nquarters; base += nwarps * 32 * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + 32 * u + lane;  // quarter index: block i/4, part i%4
      v[u] = i < nquarters ? __ldg(w + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i0 = base + 32 * u;
      const int64_t i = i0 + lane;
      const bool valid = i < nquarters;
      uint32_t m = max_magnitude8(v[u]);
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      const int bexp = static_cast<int>(m >> 7);
      const int sb = max(bexp - 2, 0);  // <= 252 for finite input
      // 2^(127 - sb) as an fp32 bit pattern (sb <= 253 keeps it finite)
      const float inv_scale = __uint_as_float(static_cast<uint32_t>(254 - min(sb, 253)) << 23);
      const uint32_t packed = encode8(v[u], inv_scale);
      if (valid) q[i] = packed;
      if (m >= 0x7F80u && valid) record_status(status, MOE_ERR_NONFINITE);
      // scale bytes: lanes 0,4,..,28 hold the scales of 8 consecutive blocks
      uint32_t lo4 = 0, hi4 = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        lo4 |= static_cast<uint32_t>(__shfl_sync(0xFFFFFFFFu, sb, 4 * b)) << (8 * b);
        hi4 |= static_cast<uint32_t>(__shfl_sync(0xFFFFFFFFu, sb, 16 + 4 * b)) << (8 * b);
      }
      const int64_t blk0 = i0 >> 2;  // multiple of 8
      if (i0 + 32 <= nquarters) {
        if (lane == 0) reinterpret_cast<uint2*>(s)[blk0 >> 3] = make_uint2(lo4, hi4);
      } else if (valid && (lane & 3) == 0) {
        s[i >> 2] = static_cast<uint8_t>(sb);
      }
    }
  }
}

}  // namespace
}  // namespace moe

extern "C" moe_status mxfp4_quantize(const uint16_t* w_bf16, int64_t rows, int64_t K,
                                     uint8_t* q_packed, uint8_t* scales, int32_t* d_status,
                                     moe_stream stream) {
  using namespace moe;
  if (rows < 0 || K < 32 || (K % 32) != 0) return MOE_ERR_SHAPE;
  if (rows > 0 && K > (int64_t(1) << 40) / rows) return MOE_ERR_SHAPE;
  if (rows == 0) return MOE_OK;
  if (!w_bf16 || !q_packed || !scales) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w_bf16) || !aligned16(q_packed) || !aligned16(scales)) return MOE_ERR_INVALID_ARG;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_device();
  if (st != MOE_OK) return st;
  const int64_t nquarters = rows * K / 8;
  int64_t want = (nquarters + kThreads * kUnroll - 1) / (kThreads * kUnroll);
  int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  const int grid = static_cast<int>(want < cap ? want : cap);
  quantize_kernel<<<grid, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint4*>(w_bf16), nquarters, reinterpret_cast<uint32_t*>(q_packed),
      scales, d_status);
  return launch_status();
}
