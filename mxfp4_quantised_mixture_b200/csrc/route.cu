// Token-choice top-k routing with the softmax taken over the chosen experts.
//
// "Welcome GPT OSS, the new open-source model family from OpenAI" (summary),
// section 4: token-choice MoE, softmax-after-topk; aitrends.kr talk summary,
// "Architecture details": 4 active experts out of 32 or 128.
//
// One warp per token.  Lane l holds logits l, l+32, ... (coalesced loads);
// k rounds of a warp arg-max on the key (logit descending, index ascending)
// pick the experts; the softmax over the k picked logits runs in fp32.
#include <math.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxPerLane = 8;  // E <= 256

// true if (va, ia) ranks before (vb, ib)
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__global__ void __launch_bounds__(kThreads) route_kernel(const float* __restrict__ logits, int T,
                                                        int E, int k, int32_t* __restrict__ idx,
                                                        float* __restrict__ w,
                                                        int32_t* __restrict__ clear_status) {
  // inside the layer the routing is the first kernel: it resets the layer's
  // device status word, which the later kernels only ever set to an error
  if (clear_status && blockIdx.x == 0 && threadIdx.x == 0) *clear_status = MOE_OK;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* row = logits + static_cast<int64_t>(t) * E;
  float v[kMaxPerLane];
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? __ldg(row + e) : -INFINITY;
  }
  unsigned taken = 0;  // bit i: slot i of this lane already chosen
  int my_idx = -1;
  float my_val = 0.f, top = 0.f;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && better(v[i], e, bv, bi)) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
      const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, off);
      if (better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    // bi stays out of range only if this lane's remaining logits are NaN
    // (a violated precondition): nothing is marked taken then
    if (bi < E && (bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (j == 0) top = bv;
    if (lane == j) {
      my_idx = bi;
      my_val = bv;
    }
  }
  const float ex = lane < k ? expf(my_val - top) : 0.f;
  float z = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xFFFFFFFFu, z, off);
  if (lane < k) {
    idx[static_cast<int64_t>(t) * k + lane] = my_idx;
    w[static_cast<int64_t>(t) * k + lane] = ex / z;
  }
}

}  // namespace

moe_status route_launch(const float* logits, int T, int E, int k, int32_t* idx, float* w,
                        int32_t* clear_status, cudaStream_t stream) {
  if (T == 0) return MOE_OK;
  const int grid = (T + kThreads / 32 - 1) / (kThreads / 32);
  return launch(route_kernel, dim3(grid), dim3(kThreads), 0, stream, logits, T, E, k, idx,
                w, clear_status);
}

}  // namespace moe

namespace moe {
moe_status router_launch(const uint16_t* x, const uint16_t* w_router, int T, int D, int E, int k,
                         float* logits, int32_t* idx, float* wts, int32_t* status,
                         cudaStream_t stream);
}  // namespace moe

extern "C" moe_status moe_route(const float* logits, int32_t T, int32_t E, int32_t k,
                                int32_t* topk_idx, float* topk_w, moe_stream stream) {
  using namespace moe;
  if (T < 0 || T > (1 << 20) || E < 1 || E > 256 || k < 1 || k > 8 || k > E) return MOE_ERR_SHAPE;
  if (T == 0) return MOE_OK;
  if (!logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(logits) || !aligned16(topk_idx) || !aligned16(topk_w)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_device();
  if (st != MOE_OK) return st;
  return route_launch(logits, T, E, k, topk_idx, topk_w, nullptr,
                      static_cast<cudaStream_t>(stream));
}
