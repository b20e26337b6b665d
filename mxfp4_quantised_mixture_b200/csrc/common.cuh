// Shared helpers of the MXFP4 MoE library (device and host side).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "moe_mxfp4.h"

namespace moe {

// ---------------------------------------------------------------- bf16 bits

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// fp32 -> bf16 bits, round to nearest even (finite inputs; NaN kept quiet)
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(f32_to_bf16_rne(lo)) |
         (static_cast<uint32_t>(f32_to_bf16_rne(hi)) << 16);
}

__device__ __forceinline__ void record_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, static_cast<int32_t>(MOE_OK), code);
}

// ------------------------------------------------------------ host helpers

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Status of the current device: MOE_OK on a compute capability 10.0 part.
moe_status check_device();

inline moe_status launch_status() {
  cudaError_t e = cudaPeekAtLastError();
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int sm_count();

bool shape_ok(const moe_shape& s);

// Launch a kernel with cudaLaunchKernelEx (argument coercion as for <<< >>>);
// with `early`, the kernel may start while the kernel before it on
// the stream still runs (once every CTA of that kernel has executed
// allow_dependents()).  Such a kernel must call wait_for_previous() before it
// reads anything the previous kernel writes; whatever the kernels before
// that one wrote is visible from its start.
template <typename... Params, typename... Args>
moe_status launch_ex(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t stream, bool early, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = early ? attr : nullptr;
  cfg.numAttrs = early ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// Launch a kernel with cudaLaunchKernelEx (argument coercion as for <<< >>>),
// in plain stream order.
template <typename... Params, typename... Args>
moe_status launch(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                  cudaStream_t stream, Args&&... args) {
  return launch_ex(kern, grid, block, smem, stream, false, std::forward<Args>(args)...);
}

// Device side of launch_ex: let the next kernel on the stream start, and
// wait until the previous kernel has completed with its writes visible (a
// no-op when this kernel was not launched early).
__device__ __forceinline__ void allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void wait_for_previous() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace moe
