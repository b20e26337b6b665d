// moe_layer_forward_static: the whole layer with its intermediates in a
// fixed-size device buffer that the library itself holds, for callers that
// cannot allocate device memory.
//
// The buffer is a file-scope __device__ array, so every GPU that loads the
// library holds MOE_STATIC_SCRATCH_BYTES of it until the process exits.  In
// host code the array's name only stands for the variable; its device address
// comes from cudaGetSymbolAddress, taken once per device (with that device
// current) on the first call made there.
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

static __device__ __align__(256) unsigned char g_layer_scratch[MOE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
void* g_ptr[kMaxDevices];
cudaError_t g_err[kMaxDevices];

void resolve(int dev) {
  void* p = nullptr;
  g_err[dev] = cudaGetSymbolAddress(&p, g_layer_scratch);
  if (g_err[dev] != cudaSuccess) {
    cudaGetLastError();
    p = nullptr;
  }
  g_ptr[dev] = p;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_layer_forward_static(const uint16_t* x, const float* logits,
                                               moe_shape shape, const uint8_t* wgu_q,
                                               const uint8_t* wgu_s, const uint8_t* wdn_q,
                                               const uint8_t* wdn_s, uint16_t* out,
                                               moe_stream stream) {
  using namespace moe;
  if (!shape_ok(shape)) return MOE_ERR_SHAPE;
  if (moe_workspace_size(shape, 2) > MOE_STATIC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
  moe_status st = check_device();
  if (st != MOE_OK) return st;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  std::call_once(g_once[dev], resolve, dev);
  if (g_ptr[dev] == nullptr) return MOE_ERR_CUDA;
  return moe_layer_forward(x, logits, shape, wgu_q, wgu_s, wdn_q, wdn_s, out, g_ptr[dev],
                           MOE_STATIC_SCRATCH_BYTES, stream);
}
