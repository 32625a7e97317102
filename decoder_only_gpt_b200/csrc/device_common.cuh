// Device helpers shared by the kernels of libgpt (storage conversions,
// warp reductions, status recording).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gpt_internal.h"

namespace gpt {

// Storage element <-> fp32.
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Record the first error of a launch sequence in the workspace status word.
__device__ __forceinline__ void record_status(int32_t* status, int32_t code, int32_t where,
                                              int64_t index) {
  if (status == nullptr) return;
  if (atomicCAS(status, 0, code) == 0) {
    gpt_device_status* s = reinterpret_cast<gpt_device_status*>(status);
    s->where = where;
    s->index = index;
  }
}

inline int last_launch_rc() { return cudaGetLastError() == cudaSuccess ? 0 : 1; }

inline int ceil_div(int64_t a, int64_t b) { return int((a + b - 1) / b); }

}  // namespace gpt
