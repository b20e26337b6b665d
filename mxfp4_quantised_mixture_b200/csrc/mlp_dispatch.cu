// The grouped expert MLP's path choice, plan and enqueue, shared by
// moe_expert_mlp, moe_expert_mlp_ex and moe_layer_forward; the tile list and
// the tensor-map encoder both GEMM paths use.
//
// "Welcome GPT OSS ..." (summary), section 4: SwiGLU experts; "Tricks from
// OpenAI gpt-oss ..." (summary), section 8: GEMMs that read the MXFP4 blocks
// and their scales directly.
#include "common.cuh"
#include "mlp_plan.cuh"

namespace moe {
namespace {

// Tile list: expert e contributes ceil(count_e / NT) tiles of up to NT rows,
// experts ascending; one CTA of 256 threads (E <= 256).
__global__ void __launch_bounds__(256) plan_tiles_kernel(const int32_t* __restrict__ offsets, int E,
                                                         int NT, Tile* __restrict__ tiles,
                                                         int* __restrict__ n_tiles,
                                                         int* __restrict__ sched, int n_sched) {
  __shared__ int base[257];
  const int e = threadIdx.x;
  for (int i = e; i < n_sched; i += blockDim.x) sched[i] = 0;
  int cnt = 0;
  if (e < E) {
    const int c = offsets[e + 1] - offsets[e];
    cnt = (c + NT - 1) / NT;
  }
  base[e + 1] = cnt;
  if (e == 0) base[0] = 0;
  __syncthreads();
  if (e == 0)
    for (int i = 1; i <= E; ++i) base[i] += base[i - 1];
  __syncthreads();
  if (e < E) {
    const int r0 = offsets[e], c = offsets[e + 1] - offsets[e];
    for (int t = 0; t < cnt; ++t) {
      Tile tl;
      tl.e = e;
      tl.row0 = r0 + t * NT;
      tl.nrows = min(NT, c - t * NT);
      tl.pad = 0;
      tiles[base[e] + t] = tl;
    }
  }
  if (e == 0) *n_tiles = base[E];
}

}  // namespace

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return static_cast<EncodeTiledFn>(nullptr);
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

moe_status plan_tiles_launch(const int32_t* offsets, int E, int NT, Tile* tiles, int* n_tiles,
                             int* sched, int n_sched, cudaStream_t stream) {
  return launch(plan_tiles_kernel, dim3(1), dim3(256), 0, stream, offsets, E, NT, tiles,
                n_tiles, sched, n_sched);
}

// Decode-sized shapes (few routed rows per expert) stream the weights once
// per small token tile and are bound by HBM: they take the block-scaled path,
// which moves the codes straight into the tensor core.  Token-heavy shapes
// are bound by the tensor core and take the decode-to-bf16 path, whose
// 2-CTA-per-SM pipeline with up to 256-token tiles keeps it busier.
int resolve_path(const moe_shape& sh, int path) {
  if (path != kPathAuto) return path;
  const int64_t S = static_cast<int64_t>(sh.T) * sh.k;
  return 2 * ((S + sh.E - 1) / sh.E) <= 64 ? kPathBlockScaled : kPathBf16Decode;
}

int mlp_tile_width(const moe_shape& sh, int path) {
  return resolve_path(sh, path) == kPathBlockScaled ? mx_tile_width(sh) : bf_tile_width(sh);
}

size_t expert_mlp_workspace(const moe_shape& sh, int path) {
  return resolve_path(sh, path) == kPathBlockScaled ? mx_workspace(sh) : bf_workspace(sh);
}

moe_status expert_mlp_plan(const moe_shape& sh, int path, const uint16_t* x_perm,
                           const uint8_t* wgu_q, const uint8_t* wgu_s, const uint8_t* wdn_q,
                           const uint8_t* wdn_s, uint16_t* h, uint16_t* y_perm, void* ws,
                           MlpPlan* plan) {
  plan->sh = sh;
  plan->path = resolve_path(sh, path);
  plan->x_perm = x_perm;
  plan->wgu_q = wgu_q;
  plan->wgu_s = wgu_s;
  plan->wdn_q = wdn_q;
  plan->wdn_s = wdn_s;
  plan->h = h;
  plan->y_perm = y_perm;
  plan->sched = nullptr;
  plan->n_sched = 0;
  if (plan->path == kPathBlockScaled) return mx_plan(plan, ws);
  if (!h) return MOE_ERR_INVALID_ARG;
  return bf_plan(plan, ws);
}

moe_status expert_mlp_enqueue(const MlpPlan& plan, const MlpInput& in, int32_t* status,
                              int fail_cta, cudaStream_t stream) {
  if (plan.sh.T == 0) return MOE_OK;
  return plan.path == kPathBlockScaled ? mx_enqueue(plan, in, status, fail_cta, stream)
                                       : bf_enqueue(plan, in, status, fail_cta, stream);
}

}  // namespace moe
