// moe_layer_forward_static: the whole layer with its intermediates in a
// fixed-size device buffer that the library itself holds, for callers that
// cannot allocate device memory.
//
// The buffer is a file-scope __device__ array, so every GPU that loads the
// library holds MOE_STATIC_SCRATCH_BYTES of it until the process exits.  In
// host code the array's name only stands for the variable; its device address
// comes from cudaGetSymbolAddress, taken per device (with that device
// current) on the first call made there that succeeds in taking it.
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

static __device__ __align__(256) unsigned char g_layer_scratch[MOE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ptr[kMaxDevices];

// The array's device address on the current device `dev`, or null when the
// lookup fails.  Only a successful lookup is kept: a failed one (for example
// one made while the stream was being captured) is tried again on the next
// call.
void* scratch_on(int dev) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_layer_scratch) != cudaSuccess) {
      cudaGetLastError();
      p = nullptr;
    }
    g_ptr[dev] = p;
  }
  return g_ptr[dev];
}

moe_status current_scratch(void** out) {
  moe_status st = check_device();
  if (st != MOE_OK) return st;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  *out = scratch_on(dev);
  return *out ? MOE_OK : MOE_ERR_CUDA;
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
  void* scratch = nullptr;
  moe_status st = current_scratch(&scratch);
  if (st != MOE_OK) return st;
  return moe_layer_forward(x, logits, shape, wgu_q, wgu_s, wdn_q, wdn_s, out, scratch,
                           MOE_STATIC_SCRATCH_BYTES, stream);
}

extern "C" moe_status moe_layer_static_status(int32_t* d_status, moe_stream stream) {
  using namespace moe;
  if (!d_status || (reinterpret_cast<uintptr_t>(d_status) & 3u)) return MOE_ERR_INVALID_ARG;
  void* scratch = nullptr;
  moe_status st = current_scratch(&scratch);
  if (st != MOE_OK) return st;
  // the layer's status word is the first 4 bytes of its workspace
  if (cudaMemcpyAsync(d_status, scratch, 4, cudaMemcpyDeviceToDevice,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
