// Element-wise GEMM epilogues shared by the GEMM kernels.  The per-row
// cross-entropy statistics (EPI_CE_FWD) need a row reduction across the tile
// and are implemented inside each GEMM kernel.
#pragma once

#include "device_common.cuh"

namespace gpt {

template <typename T>
__device__ __forceinline__ void epi_elem(const GemmArgs& g, int m, int n, float acc) {
  const int64_t idx = int64_t(m) * g.ldo + n;
  switch (g.epi) {
    case EPI_STORE: {
      T* o = static_cast<T*>(g.out) + idx;
      *o = from_f<T>(g.beta ? to_f(*o) + acc : acc);
      break;
    }
    case EPI_STORE_F32:
      static_cast<float*>(g.out)[idx] = acc;
      break;
    case EPI_RESID_F32:
      static_cast<float*>(g.out)[idx] += acc;
      break;
    case EPI_RELU2: {
      float r = fmaxf(acc, 0.f);
      static_cast<T*>(g.out)[idx] = from_f<T>(r * r);
      break;
    }
    case EPI_DRELU2: {
      // relu(u)^2' = 2 relu(u) = 2 sqrt(a) with a = relu(u)^2 the stored activation
      float a = to_f(static_cast<const T*>(g.aux)[idx]);
      static_cast<T*>(g.out)[idx] = from_f<T>(acc * 2.f * sqrtf(a));
      break;
    }
    case EPI_CE_BWD: {
      float v = 0.f;
      if (n < g.n_valid) {
        float p = expf(acc - g.lse[m]);
        v = (p - (n == g.targets[m] ? 1.f : 0.f)) * g.inv_n;
      }
      static_cast<T*>(g.out)[idx] = from_f<T>(v);
      break;
    }
    default:
      break;
  }
}

}  // namespace gpt
