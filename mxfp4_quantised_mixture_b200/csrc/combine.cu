// Routing-weighted combine as a deterministic gather-sum.
//
// "Welcome GPT OSS, the new open-source model family from OpenAI" (summary),
// section 4: the chosen experts' outputs are mixed with the softmax weights
// taken over the chosen experts.
//
// out[t][d] = bf16( sum_{j ascending} w[t][j] * y_perm[slot_pos[t*k + j]][d] )
// with fp32 accumulation.  Each thread owns 8 consecutive d of one token
// (16-byte loads of the k expert rows, one 16-byte store); the k rows are
// read in the fixed order j = 0..k-1, so the result does not depend on
// scheduling.  HBM-bound: (k + 1) * 2 bytes per output element.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) combine_kernel(const uint4* __restrict__ y,
                                                          const int32_t* __restrict__ slot_pos,
                                                          const float* __restrict__ w, int64_t T,
                                                          int k, int vec_per_row,
                                                          uint4* __restrict__ out) {
  const int64_t n = T * vec_per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t t = i / vec_per_row;
    const int v = static_cast<int>(i - t * vec_per_row);
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int32_t p = __ldg(slot_pos + t * k + j);
      if (p < 0) continue;
      const float wj = __ldg(w + t * k + j);
      const uint4 r = __ldg(y + static_cast<int64_t>(p) * vec_per_row + v);
      const uint32_t rr[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] = fmaf(wj, __uint_as_float(rr[q] << 16), acc[2 * q]);
        acc[2 * q + 1] = fmaf(wj, __uint_as_float(rr[q] & 0xFFFF0000u), acc[2 * q + 1]);
      }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    out[i] = o;
  }
}

}  // namespace

moe_status combine_launch(const uint16_t* y_perm, const int32_t* slot_pos, const float* w,
                          const moe_shape& sh, uint16_t* out, cudaStream_t stream) {
  if (sh.T == 0) return MOE_OK;
  const int vec = sh.d_model / 8;
  const int64_t n = static_cast<int64_t>(sh.T) * vec;
  int64_t want = (n + kThreads - 1) / kThreads;
  int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  const int grid = static_cast<int>(want < cap ? want : cap);
  return launch(combine_kernel, dim3(grid), dim3(kThreads), 0, stream,
                reinterpret_cast<const uint4*>(y_perm), slot_pos, w, static_cast<int64_t>(sh.T),
                sh.k, vec, reinterpret_cast<uint4*>(out));
}

}  // namespace moe

extern "C" moe_status moe_combine(const uint16_t* y_perm, const int32_t* slot_pos,
                                  const float* topk_w, moe_shape shape, uint16_t* out,
                                  moe_stream stream) {
  using namespace moe;
  if (!shape_ok(shape)) return MOE_ERR_SHAPE;
  if (shape.T == 0) return MOE_OK;
  if (!y_perm || !slot_pos || !topk_w || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(slot_pos) || !aligned16(topk_w) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  moe_status st = check_device();
  if (st != MOE_OK) return st;
  return combine_launch(y_perm, slot_pos, topk_w, shape, out, static_cast<cudaStream_t>(stream));
}
