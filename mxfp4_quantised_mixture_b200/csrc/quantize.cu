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
// bytes plus 8 contiguous scale bytes.  The kernel is a grid-stride stream,
// bound by HBM (2 bytes read, 17/32 byte written per element).
#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t encode8(uint4 v, float inv_scale) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t b = (w[i >> 1] >> ((i & 1) * 16)) & 0xFFFFu;
    // |x| / scale is exact: bf16 magnitude times a power of two
    const float r = __uint_as_float((b & 0x7FFFu) << 16) * inv_scale;
    // round to nearest, ties to the even mantissa bit, saturate at 6
    uint32_t c = (r > 0.25f) + (r >= 0.75f) + (r > 1.25f) + (r >= 1.75f) + (r > 2.5f) +
                 (r >= 3.5f) + (r > 5.0f);
    c |= (b >> 12) & 8u;  // sign bit
    out |= c << (4 * i);
  }
  return out;
}

__global__ void __launch_bounds__(kThreads) quantize_kernel(const uint4* __restrict__ w,
                                                           int64_t nquarters,
                                                           uint32_t* __restrict__ q,
                                                           uint8_t* __restrict__ s,
                                                           int32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  for (int64_t base = warp0 * 32; base < nquarters; base += nwarps * 32) {
    const int64_t i = base + lane;  // quarter index: block i/4, part i%4
    const bool valid = i < nquarters;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (valid) v = __ldg(w + i);
    // magnitude bits order like the values for finite bf16
    uint32_t m = 0, nonfinite = 0;
    const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = ww[j] & 0x7FFFu, hi = (ww[j] >> 16) & 0x7FFFu;
      m = max(m, max(lo, hi));
      nonfinite |= ((lo & 0x7F80u) == 0x7F80u) | ((hi & 0x7F80u) == 0x7F80u);
    }
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    const int bexp = static_cast<int>(m >> 7);
    const int sb = max(bexp - 2, 0);  // <= 252 for finite input
    // 2^(127 - sb) as an fp32 bit pattern (sb <= 253 keeps it finite)
    const float inv_scale = __uint_as_float(static_cast<uint32_t>(254 - min(sb, 253)) << 23);
    const uint32_t packed = encode8(v, inv_scale);
    if (valid) q[i] = packed;
    if (nonfinite && valid) record_status(status, MOE_ERR_NONFINITE);
    // scale bytes: lanes 0,4,..,28 hold the scales of 8 consecutive blocks
    uint32_t lo4 = 0, hi4 = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      lo4 |= static_cast<uint32_t>(__shfl_sync(0xFFFFFFFFu, sb, 4 * b)) << (8 * b);
      hi4 |= static_cast<uint32_t>(__shfl_sync(0xFFFFFFFFu, sb, 16 + 4 * b)) << (8 * b);
    }
    const int64_t blk0 = base >> 2;  // multiple of 8
    if (base + 32 <= nquarters) {
      if (lane == 0) reinterpret_cast<uint2*>(s)[blk0 >> 3] = make_uint2(lo4, hi4);
    } else if (valid && (lane & 3) == 0) {
      s[i >> 2] = static_cast<uint8_t>(sb);
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
  int64_t want = (nquarters + kThreads - 1) / kThreads;
  int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  const int grid = static_cast<int>(want < cap ? want : cap);
  quantize_kernel<<<grid, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint4*>(w_bf16), nquarters, reinterpret_cast<uint32_t*>(q_packed),
      scales, d_status);
  return launch_status();
}
