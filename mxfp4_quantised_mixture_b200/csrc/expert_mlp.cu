// Grouped SwiGLU expert MLP on MXFP4 weights (first, CUDA-core version).
//
// "Welcome GPT OSS ..." (summary), section 4: SwiGLU experts;
// "Tricks from OpenAI gpt-oss ..." (summary), section 8: GEMMs that read the
// 32-element blocks and their scales; aitrends.kr talk summary, "Hardware
// optimisation": weights stay 4-bit in memory and are raised to higher
// precision only for the arithmetic.
//
// Kernel 1 (gate/up + SwiGLU): one warp per output feature n of one expert;
// it streams gate row n and up row F+n once per chunk of 8 token rows, each
// lane decoding 8 consecutive elements (4 code bytes, one scale) and
// multiplying them with the 8 rows; h = bf16(silu(g) * u).
// Kernel 2 (down): one warp per output feature d, reducing over F.
// Products are exact in fp32 (a 2-bit-significand weight times a bf16), and
// the sums accumulate in fp32.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kRows = 8;

__device__ __forceinline__ void decode8(uint32_t codes, uint8_t sbyte, float* out) {
  // E2M1 magnitudes of codes 0..7
  const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
  // 2^(sbyte - 127): normal for sbyte >= 1, the fp32 subnormal 2^-127 for 0
  const float scale = sbyte ? __uint_as_float(static_cast<uint32_t>(sbyte) << 23)
                            : __uint_as_float(0x00400000u);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t c = (codes >> (4 * i)) & 15u;
    const float v = mag[c & 7] * scale;
    out[i] = (c & 8) ? -v : v;
  }
}

__device__ __forceinline__ void unpack8(uint4 r, float* out) {
  const uint32_t rr[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    out[2 * q] = __uint_as_float(rr[q] << 16);
    out[2 * q + 1] = __uint_as_float(rr[q] & 0xFFFF0000u);
  }
}

__global__ void __launch_bounds__(kWarps * 32) gate_up_simt_kernel(
    const uint16_t* __restrict__ x_perm, const int32_t* __restrict__ offsets, int D, int F,
    const uint8_t* __restrict__ wq, const uint8_t* __restrict__ ws, uint16_t* __restrict__ h) {
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int e = blockIdx.y;
  if (n >= F) return;
  const int r0 = __ldg(offsets + e), r1 = __ldg(offsets + e + 1);
  const int64_t grow = static_cast<int64_t>(e) * 2 * F + n;  // gate row; up row is +F
  const uint8_t* gq = wq + grow * (D / 2);
  const uint8_t* uq = wq + (grow + F) * (D / 2);
  const uint8_t* gs = ws + grow * (D / 32);
  const uint8_t* us = ws + (grow + F) * (D / 32);
  for (int r = r0; r < r1; r += kRows) {
    float ag[kRows], au[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) ag[i] = au[i] = 0.f;
    for (int kk = lane * 8; kk < D; kk += 256) {
      float wg[8], wu[8];
      decode8(__ldg(reinterpret_cast<const uint32_t*>(gq + kk / 2)), __ldg(gs + kk / 32), wg);
      decode8(__ldg(reinterpret_cast<const uint32_t*>(uq + kk / 2)), __ldg(us + kk / 32), wu);
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        if (r + i >= r1) break;
        float xv[8];
        unpack8(__ldg(reinterpret_cast<const uint4*>(x_perm + static_cast<int64_t>(r + i) * D + kk)),
                xv);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          ag[i] = fmaf(wg[q], xv[q], ag[i]);
          au[i] = fmaf(wu[q], xv[q], au[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        ag[i] += __shfl_xor_sync(0xFFFFFFFFu, ag[i], off);
        au[i] += __shfl_xor_sync(0xFFFFFFFFu, au[i], off);
      }
    }
    if (lane < kRows && r + lane < r1) {
      float g = 0.f, u = 0.f;
#pragma unroll
      for (int i = 0; i < kRows; ++i)
        if (i == lane) {
          g = ag[i];
          u = au[i];
        }
      const float silu = g / (1.f + expf(-g));
      h[static_cast<int64_t>(r + lane) * F + n] = f32_to_bf16_rne(silu * u);
    }
  }
}

__global__ void __launch_bounds__(kWarps * 32) down_simt_kernel(
    const uint16_t* __restrict__ h, const int32_t* __restrict__ offsets, int D, int F,
    const uint8_t* __restrict__ wq, const uint8_t* __restrict__ ws, uint16_t* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int d = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int e = blockIdx.y;
  if (d >= D) return;
  const int r0 = __ldg(offsets + e), r1 = __ldg(offsets + e + 1);
  const int64_t row = static_cast<int64_t>(e) * D + d;
  const uint8_t* dq = wq + row * (F / 2);
  const uint8_t* ds = ws + row * (F / 32);
  for (int r = r0; r < r1; r += kRows) {
    float acc[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) acc[i] = 0.f;
    for (int kk = lane * 8; kk < F; kk += 256) {
      float wd[8];
      decode8(__ldg(reinterpret_cast<const uint32_t*>(dq + kk / 2)), __ldg(ds + kk / 32), wd);
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        if (r + i >= r1) break;
        float hv[8];
        unpack8(__ldg(reinterpret_cast<const uint4*>(h + static_cast<int64_t>(r + i) * F + kk)), hv);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[i] = fmaf(wd[q], hv[q], acc[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < kRows; ++i)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], off);
    if (lane < kRows && r + lane < r1) {
      float a = 0.f;
#pragma unroll
      for (int i = 0; i < kRows; ++i)
        if (i == lane) a = acc[i];
      y[static_cast<int64_t>(r + lane) * D + d] = f32_to_bf16_rne(a);
    }
  }
}

}  // namespace

size_t expert_mlp_workspace(const moe_shape& sh) {
  (void)sh;
  return 256;
}

moe_status expert_mlp_launch(const uint16_t* x_perm, const int32_t* offsets, const moe_shape& sh,
                             const uint8_t* wgu_q, const uint8_t* wgu_s, const uint8_t* wdn_q,
                             const uint8_t* wdn_s, uint16_t* h, uint16_t* y_perm, void* ws,
                             cudaStream_t stream) {
  (void)ws;
  if (sh.T == 0) return MOE_OK;
  dim3 g1((sh.d_ff + kWarps - 1) / kWarps, sh.E);
  gate_up_simt_kernel<<<g1, kWarps * 32, 0, stream>>>(x_perm, offsets, sh.d_model, sh.d_ff, wgu_q,
                                                      wgu_s, h);
  moe_status st = launch_status();
  if (st != MOE_OK) return st;
  dim3 g2((sh.d_model + kWarps - 1) / kWarps, sh.E);
  down_simt_kernel<<<g2, kWarps * 32, 0, stream>>>(h, offsets, sh.d_model, sh.d_ff, wdn_q, wdn_s,
                                                   y_perm);
  return launch_status();
}

}  // namespace moe
