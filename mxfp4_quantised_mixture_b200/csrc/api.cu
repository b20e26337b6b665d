// C ABI entry points that orchestrate the layer, validate arguments and lay
// out the caller-owned workspace.
//
// moe_layer_forward enqueues, on one stream, the layer as the pages describe
// it: token-choice top-k with softmax over the chosen experts ("Welcome
// GPT OSS ..." (summary), section 4), grouping of the routed tokens by
// expert, the SwiGLU experts on MXFP4 weights ("Tricks from OpenAI gpt-oss
// ..." (summary), sections 6 and 8), and the weighted combine.
#include <mutex>

#include "common.cuh"
#include "mlp_plan.cuh"

namespace moe {

moe_status route_launch(const float* logits, int T, int E, int k, int32_t* idx, float* w,
                        int32_t* clear_status, cudaStream_t stream);
moe_status permute_launch(const int32_t* idx, const uint16_t* x, const moe_shape& sh,
                          int32_t* counts, int32_t* offsets, int32_t* sorted_slot,
                          int32_t* slot_pos, uint16_t* x_perm, int NT, Tile* tiles,
                          int* n_tiles, int* sched, int n_sched, cudaStream_t stream);
moe_status combine_launch(const uint16_t* y_perm, const int32_t* slot_pos, const float* w,
                          const moe_shape& sh, uint16_t* out, cudaStream_t stream);
size_t unquantised_workspace(const moe_shape& sh);
moe_status unquantised_mlp(const uint16_t* x_perm, const int32_t* offsets, const moe_shape& sh,
                           const uint16_t* w_gu, const uint16_t* w_dn, uint16_t* h,
                           uint16_t* y_perm, void* ws, int32_t* status, cudaStream_t stream);

namespace {

constexpr int kMaxDevices = 64;
std::once_flag g_dev_once[kMaxDevices];
moe_status g_dev_status[kMaxDevices];
int g_dev_sms[kMaxDevices];

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return dev;
}

void probe_device(int dev) {
  int major = 0, minor = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    g_dev_status[dev] = MOE_ERR_CUDA;
    return;
  }
  g_dev_sms[dev] = sms;
  g_dev_status[dev] = (major == 10 && minor == 0) ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

// Workspace of moe_layer_forward: every intermediate, 256-byte aligned.
struct LayerWs {
  size_t status, idx, w, counts, offsets, sorted_slot, slot_pos, x_perm, h, y_perm, mlp, total;
};

LayerWs layer_ws(const moe_shape& s) {
  const size_t S = static_cast<size_t>(s.T) * s.k;
  LayerWs L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  L.status = take(256);
  L.idx = take(S * 4);
  L.w = take(S * 4);
  L.counts = take(static_cast<size_t>(s.E) * 4);
  L.offsets = take(static_cast<size_t>(s.E + 1) * 4);
  L.sorted_slot = take(S * 4);
  L.slot_pos = take(S * 4);
  // the block-scaled path splits its rows straight from x and hands h to the
  // down GEMM as pieces: neither x_perm nor h is written there
  const bool block_scaled = resolve_path(s, kPathAuto) == kPathBlockScaled;
  L.x_perm = take(block_scaled ? 0 : S * s.d_model * 2);
  L.h = take(block_scaled ? 0 : S * s.d_ff * 2);
  L.y_perm = take(S * s.d_model * 2);
  L.mlp = take(expert_mlp_workspace(s, kPathAuto));
  L.total = o;
  return L;
}

}  // namespace

moe_status check_device() {
  const int dev = current_device();
  if (dev < 0) return MOE_ERR_CUDA;
  if (dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::call_once(g_dev_once[dev], probe_device, dev);
  return g_dev_status[dev];
}

int sm_count() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  std::call_once(g_dev_once[dev], probe_device, dev);
  return g_dev_sms[dev] > 0 ? g_dev_sms[dev] : 148;
}

// status head of the standalone expert-MLP workspace
constexpr size_t kMlpStatusBytes = 256;

bool shape_ok(const moe_shape& s) {
  if (s.T < 0 || s.T > (1 << 20)) return false;
  if (s.E < 1 || s.E > 256) return false;
  if (s.k < 1 || s.k > 8 || s.k > s.E) return false;
  if (s.d_model < 128 || s.d_model > 16384 || (s.d_model % 64) != 0) return false;
  if (s.d_ff < 128 || s.d_ff > 16384 || (s.d_ff % 64) != 0) return false;
  if (static_cast<int64_t>(s.T) * s.k >= (int64_t(1) << 31)) return false;
  return true;
}

}  // namespace moe

extern "C" {

size_t moe_workspace_size(moe_shape shape, int which) {
  using namespace moe;
  if (!shape_ok(shape)) return 0;
  switch (which) {
    case 0:
      return 0;
    case 1:
      return kMlpStatusBytes + expert_mlp_workspace(shape, kPathAuto);
    case 2:
      return layer_ws(shape).total;
    case 3:
      return kMlpStatusBytes + expert_mlp_workspace(shape, kPathBlockScaled);
    case 4:
      return kMlpStatusBytes + expert_mlp_workspace(shape, kPathBf16Decode);
    case 5:
      return kMlpStatusBytes + unquantised_workspace(shape);
    default:
      return 0;
  }
}

const char* moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK:
      return "MOE_OK";
    case MOE_ERR_INVALID_ARG:
      return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_SHAPE:
      return "MOE_ERR_SHAPE";
    case MOE_ERR_WORKSPACE:
      return "MOE_ERR_WORKSPACE";
    case MOE_ERR_UNSUPPORTED:
      return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_CUDA:
      return "MOE_ERR_CUDA";
    case MOE_ERR_NONFINITE:
      return "MOE_ERR_NONFINITE";
    case MOE_ERR_TIMEOUT:
      return "MOE_ERR_TIMEOUT";
  }
  return "MOE_ERR_UNKNOWN";
}

moe_status moe_expert_mlp_ex(const uint16_t* x_perm, const int32_t* offsets, moe_shape shape,
                             const uint8_t* wgu_q, const uint8_t* wgu_s, const uint8_t* wdn_q,
                             const uint8_t* wdn_s, uint16_t* h, uint16_t* y_perm, void* ws,
                             size_t ws_bytes, int32_t path, int32_t test_timeout_cta,
                             moe_stream stream) {
  using namespace moe;
  if (!shape_ok(shape)) return MOE_ERR_SHAPE;
  if (path != kPathAuto && path != kPathBlockScaled && path != kPathBf16Decode)
    return MOE_ERR_INVALID_ARG;
  if (shape.T == 0) return MOE_OK;
  const void* ptrs[] = {x_perm, offsets, wgu_q, wgu_s, wdn_q, wdn_s, h, y_perm};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (!aligned32(wgu_q) || !aligned32(wdn_q)) return MOE_ERR_INVALID_ARG;
  // the first kMlpStatusBytes of ws hold the device status word, the rest
  // is the GEMMs' workspace (same alignment class as ws itself)
  const size_t need = kMlpStatusBytes + expert_mlp_workspace(shape, path);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  moe_status st = check_device();
  if (st != MOE_OK) return st;
  MlpPlan plan;
  if ((st = expert_mlp_plan(shape, path, x_perm, wgu_q, wgu_s, wdn_q, wdn_s, h, y_perm,
                            static_cast<char*>(ws) + kMlpStatusBytes, &plan)) != MOE_OK)
    return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  MlpInput in{};
  in.offsets = offsets;
  return expert_mlp_enqueue(plan, in, static_cast<int32_t*>(ws), test_timeout_cta < 0 ? -1 : test_timeout_cta, s);
}

moe_status moe_expert_mlp(const uint16_t* x_perm, const int32_t* offsets, moe_shape shape,
                          const uint8_t* wgu_q, const uint8_t* wgu_s, const uint8_t* wdn_q,
                          const uint8_t* wdn_s, uint16_t* h, uint16_t* y_perm, void* ws,
                          size_t ws_bytes, moe_stream stream) {
  return moe_expert_mlp_ex(x_perm, offsets, shape, wgu_q, wgu_s, wdn_q, wdn_s, h, y_perm, ws,
                           ws_bytes, MOE_MLP_PATH_AUTO, -1, stream);
}

moe_status moe_expert_mlp_unquantised(const uint16_t* x_perm, const int32_t* offsets,
                                      moe_shape shape, const uint16_t* w_gu, const uint16_t* w_dn,
                                      uint16_t* h, uint16_t* y_perm, void* ws, size_t ws_bytes,
                                      moe_stream stream) {
  using namespace moe;
  if (!shape_ok(shape)) return MOE_ERR_SHAPE;
  if (shape.T == 0) return MOE_OK;
  const void* ptrs[] = {x_perm, offsets, w_gu, w_dn, h, y_perm};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const size_t need = kMlpStatusBytes + unquantised_workspace(shape);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  moe_status st = check_device();
  if (st != MOE_OK) return st;
  return unquantised_mlp(x_perm, offsets, shape, w_gu, w_dn, h, y_perm,
                         static_cast<char*>(ws) + kMlpStatusBytes, static_cast<int32_t*>(ws),
                         static_cast<cudaStream_t>(stream));
}

moe_status moe_layer_forward(const uint16_t* x, const float* logits, moe_shape shape,
                             const uint8_t* wgu_q, const uint8_t* wgu_s, const uint8_t* wdn_q,
                             const uint8_t* wdn_s, uint16_t* out, void* ws, size_t ws_bytes,
                             moe_stream stream) {
  using namespace moe;
  if (!shape_ok(shape)) return MOE_ERR_SHAPE;
  if (shape.T == 0) return MOE_OK;
  const void* ptrs[] = {x, logits, wgu_q, wgu_s, wdn_q, wdn_s, out};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (!aligned32(wgu_q) || !aligned32(wdn_q)) return MOE_ERR_INVALID_ARG;
  const LayerWs L = layer_ws(shape);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  moe_status st = check_device();
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(ws);
  auto at = [&](size_t off) { return static_cast<void*>(base + off); };
  int32_t* status = static_cast<int32_t*>(at(L.status));
  int32_t* idx = static_cast<int32_t*>(at(L.idx));
  float* w = static_cast<float*>(at(L.w));
  int32_t* counts = static_cast<int32_t*>(at(L.counts));
  int32_t* offsets = static_cast<int32_t*>(at(L.offsets));
  int32_t* sorted_slot = static_cast<int32_t*>(at(L.sorted_slot));
  int32_t* slot_pos = static_cast<int32_t*>(at(L.slot_pos));
  uint16_t* x_perm = static_cast<uint16_t*>(at(L.x_perm));
  uint16_t* h = static_cast<uint16_t*>(at(L.h));
  uint16_t* y_perm = static_cast<uint16_t*>(at(L.y_perm));
  // everything that can refuse the call happens here, before the first launch
  MlpPlan plan;
  const bool block_scaled = resolve_path(shape, kPathAuto) == kPathBlockScaled;
  if ((st = expert_mlp_plan(shape, kPathAuto, x_perm, wgu_q, wgu_s, wdn_q, wdn_s,
                            block_scaled ? nullptr : h, y_perm, at(L.mlp), &plan)) != MOE_OK)
    return st;
  const int NT = mlp_tile_width(shape, kPathAuto);
  // route (its first thread also clears the status word), then permute with
  // the GEMMs' tile list; the block-scaled path splits its rows straight from
  // x, so only the other path gathers x_perm
  if ((st = route_launch(logits, shape.T, shape.E, shape.k, idx, w, status, s)) != MOE_OK)
    return st;
  if ((st = permute_launch(idx, x, shape, counts, offsets, sorted_slot, slot_pos,
                           block_scaled ? nullptr : x_perm, NT, plan.tiles, plan.n_tiles,
                           plan.sched, plan.n_sched, s)) != MOE_OK)
    return st;
  MlpInput in{};
  in.offsets = offsets;
  in.tiles_ready = true;
  if (block_scaled) {
    in.x = x;
    in.sorted_slot = sorted_slot;
    in.k = shape.k;
  }
  if ((st = expert_mlp_enqueue(plan, in, status, -1, s)) != MOE_OK) return st;
  return combine_launch(y_perm, slot_pos, w, shape, out, s);
}

}  // extern "C"
