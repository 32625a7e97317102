// Element-wise parts of the optimizer step: AdamW for the embedding and
// lm_head, and Muon's momentum, Frobenius normalisation, NorMuon row rescale
// and update for the block matrices ("ChatGPT'nizi 50 Dolara Nasil
// Egitirsiniz?", section "2. Muon Optimize Edici (nanochat/optim.py)", and its
// "NorMuon Varyans Azaltma" lines).  The Newton-Schulz products between
// the normalisation and the update run on the tensor-core GEMM (EPI_AXPBY).
//
// All kernels are HBM-bound streams over 8-element groups (16-byte bf16 and
// 2 x 16-byte fp32 accesses); n is a multiple of 8 for every tensor (d_model is
// a multiple of 64).  The sum of squares uses a fixed grid and a fixed
// reduction order, so every step is deterministic.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "device_common.cuh"
#include "gpt_internal.h"

namespace gpt {
namespace {

__device__ __forceinline__ void load8_bf16(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void store8_bf16(__nv_bfloat16* p, const float (&f)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ void load8_f32(const float* p, float (&f)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void store8_f32(float* p, const float (&f)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

__global__ void optim_init_kernel(const __nv_bfloat16* __restrict__ p, float* __restrict__ w,
                                  float* __restrict__ m, float* __restrict__ v, int64_t n8) {
  const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += int64_t(gridDim.x) * blockDim.x) {
    float f[8];
    load8_bf16(p + 8 * i, f);
    store8_f32(w + 8 * i, f);
    store8_f32(m + 8 * i, z);
    store8_f32(v + 8 * i, z);
  }
}

// AdamW with bias correction (bc1 = 1 - b1^t, bc2 = 1 - b2^t) and decoupled
// weight decay; the bf16 parameters are rewritten from the fp32 master.
__global__ void adamw_kernel(__nv_bfloat16* __restrict__ p, const __nv_bfloat16* __restrict__ g,
                             float* __restrict__ w, float* __restrict__ m, float* __restrict__ v,
                             int64_t n8, float lr, float b1, float b2, float eps, float wd,
                             float bc1, float bc2) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += int64_t(gridDim.x) * blockDim.x) {
    float gf[8], mf[8], vf[8], wf[8];
    load8_bf16(g + 8 * i, gf);
    load8_f32(m + 8 * i, mf);
    load8_f32(v + 8 * i, vf);
    load8_f32(w + 8 * i, wf);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      mf[e] = b1 * mf[e] + (1.f - b1) * gf[e];
      vf[e] = b2 * vf[e] + (1.f - b2) * gf[e] * gf[e];
      wf[e] = wf[e] * (1.f - lr * wd) - lr * (mf[e] / bc1) / (sqrtf(vf[e] / bc2) + eps);
    }
    store8_f32(m + 8 * i, mf);
    store8_f32(v + 8 * i, vf);
    store8_f32(w + 8 * i, wf);
    store8_bf16(p + 8 * i, wf);
  }
}

// Muon momentum: M = mu M + G, U = G + mu M (Nesterov) or M; per-block sum of
// U^2 in a fixed order.
__global__ void muon_momentum_kernel(const __nv_bfloat16* __restrict__ g, float* __restrict__ mom,
                                     int64_t n8, float mu, int nesterov, float* __restrict__ partial) {
  float s = 0.f;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += int64_t(gridDim.x) * blockDim.x) {
    float gf[8], mf[8];
    load8_bf16(g + 8 * i, gf);
    load8_f32(mom + 8 * i, mf);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      mf[e] = mu * mf[e] + gf[e];
      const float u = nesterov ? gf[e] + mu * mf[e] : mf[e];
      s += u * u;
    }
    store8_f32(mom + 8 * i, mf);
  }
  __shared__ float red[32];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < blockDim.x / 32 ? red[threadIdx.x] : 0.f;
    t = warp_sum(t);
    if (threadIdx.x == 0) partial[blockIdx.x] = t;
  }
}

// inv = 1 / (sqrt(sum of the partials, in block order) + 1e-7), in partial[nb]
__global__ void muon_norm_kernel(float* __restrict__ partial, int nb) {
  float s = 0.f;
  for (int i = threadIdx.x; i < nb; i += 32) s += partial[i];
  s = warp_sum(s);
  if (threadIdx.x == 0) partial[nb] = 1.f / (sqrtf(s) + 1e-7f);
}

// x = bf16(U * inv), U recomputed from G and the updated momentum
__global__ void muon_scale_kernel(const __nv_bfloat16* __restrict__ g, const float* __restrict__ mom,
                                  int64_t n8, float mu, int nesterov, const float* __restrict__ inv,
                                  __nv_bfloat16* __restrict__ x) {
  const float sc = *inv;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += int64_t(gridDim.x) * blockDim.x) {
    float gf[8], mf[8], u[8];
    load8_bf16(g + 8 * i, gf);
    load8_f32(mom + 8 * i, mf);
#pragma unroll
    for (int e = 0; e < 8; ++e) u[e] = (nesterov ? gf[e] + mu * mf[e] : mf[e]) * sc;
    store8_bf16(x + 8 * i, u);
  }
}

__global__ void muon_apply_kernel(const __nv_bfloat16* __restrict__ x, float* __restrict__ w,
                                  __nv_bfloat16* __restrict__ p, int64_t n8, float step) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += int64_t(gridDim.x) * blockDim.x) {
    float xf[8], wf[8];
    load8_bf16(x + 8 * i, xf);
    load8_f32(w + 8 * i, wf);
#pragma unroll
    for (int e = 0; e < 8; ++e) wf[e] -= step * xf[e];
    store8_f32(w + 8 * i, wf);
    store8_bf16(p + 8 * i, wf);
  }
}

// NorMuon, per row r of one orthogonalised update X [rows, cols] (bf16):
// v_mean = mean_c X[r,c]^2; buf = beta2 buf + (1 - beta2) v_mean (the per-row
// state); step = 1 / sqrt(max(buf, 1e-10)).  One warp per row, a fixed
// lane-strided order.
__global__ void normuon_rows_kernel(const __nv_bfloat16* __restrict__ x, float* __restrict__ buf,
                                    int rows, int cols, float beta2, float* __restrict__ vmean,
                                    float* __restrict__ step) {
  const int r = int(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  if (r >= rows) return;
  const __nv_bfloat16* row = x + int64_t(r) * cols;
  float s = 0.f;
  for (int c = threadIdx.x & 31; c < cols; c += 32) {
    const float v = __bfloat162float(row[c]);
    s += v * v;
  }
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) {
    const float vm = s / float(cols);
    const float b = beta2 * buf[r] + (1.f - beta2) * vm;
    buf[r] = b;
    vmean[r] = vm;
    step[r] = 1.f / sqrtf(fmaxf(b, 1e-10f));
  }
}

// The matrix-wide factor v_norm / max(v_norm_new, 1e-10) with v_norm^2 =
// sum_r v_mean[r] and v_norm_new^2 = sum_r v_mean[r] step[r]^2 (one block, a
// fixed summation order), folded into step[r] in place: the row factors.
__global__ void normuon_scale_kernel(const float* __restrict__ vmean, float* __restrict__ step,
                                     int rows) {
  __shared__ float red[2][32];
  float s1 = 0.f, s2 = 0.f;
  for (int r = threadIdx.x; r < rows; r += blockDim.x) {
    s1 += vmean[r];
    s2 += vmean[r] * step[r] * step[r];
  }
  s1 = warp_sum(s1);
  s2 = warp_sum(s2);
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x / 32] = s1;
    red[1][threadIdx.x / 32] = s2;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const bool in = threadIdx.x < blockDim.x / 32;
    s1 = warp_sum(in ? red[0][threadIdx.x] : 0.f);
    s2 = warp_sum(in ? red[1][threadIdx.x] : 0.f);
    if (threadIdx.x == 0) red[0][0] = sqrtf(s1) / fmaxf(sqrtf(s2), 1e-10f);
  }
  __syncthreads();
  const float scale = red[0][0];
  for (int r = threadIdx.x; r < rows; r += blockDim.x) step[r] *= scale;
}

// master -= step * factor[row] * x; params = bf16(master)
__global__ void muon_apply_rows_kernel(const __nv_bfloat16* __restrict__ x, float* __restrict__ w,
                                       __nv_bfloat16* __restrict__ p, int64_t n8, int cols,
                                       float step, const float* __restrict__ factor) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += int64_t(gridDim.x) * blockDim.x) {
    float xf[8], wf[8];
    load8_bf16(x + 8 * i, xf);
    load8_f32(w + 8 * i, wf);
#pragma unroll
    for (int e = 0; e < 8; ++e) wf[e] -= step * factor[(8 * i + e) / cols] * xf[e];
    store8_f32(w + 8 * i, wf);
    store8_bf16(p + 8 * i, wf);
  }
}

int stream_grid(int64_t n8) {
  const int64_t want = (n8 + 255) / 256;
  return int(want < 148 * 8 ? (want > 0 ? want : 1) : 148 * 8);
}

}  // namespace

int launch_optim_init(const void* params, float* master, float* m, float* v, int64_t n, void* stream) {
  if (n % 8) return 1;
  optim_init_kernel<<<stream_grid(n / 8), 256, 0, (cudaStream_t)stream>>>(
      static_cast<const __nv_bfloat16*>(params), master, m, v, n / 8);
  return last_launch_rc();
}

int launch_adamw(void* params, const void* grads, float* master, float* m, float* v, int64_t n,
                 float lr, float b1, float b2, float eps, float wd, float bc1, float bc2, void* stream) {
  if (n % 8) return 1;
  adamw_kernel<<<stream_grid(n / 8), 256, 0, (cudaStream_t)stream>>>(
      static_cast<__nv_bfloat16*>(params), static_cast<const __nv_bfloat16*>(grads), master, m, v,
      n / 8, lr, b1, b2, eps, wd, bc1, bc2);
  return last_launch_rc();
}

int launch_muon_prepare(const void* grads, float* mom, int64_t n, float mu, int nesterov,
                        float* partial, void* x_out, void* stream) {
  if (n % 8) return 1;
  cudaStream_t st = (cudaStream_t)stream;
  const __nv_bfloat16* g = static_cast<const __nv_bfloat16*>(grads);
  muon_momentum_kernel<<<kOptNormBlocks, 256, 0, st>>>(g, mom, n / 8, mu, nesterov, partial);
  muon_norm_kernel<<<1, 32, 0, st>>>(partial, kOptNormBlocks);
  muon_scale_kernel<<<stream_grid(n / 8), 256, 0, st>>>(g, mom, n / 8, mu, nesterov,
                                                        partial + kOptNormBlocks,
                                                        static_cast<__nv_bfloat16*>(x_out));
  return last_launch_rc();
}

int launch_muon_apply(const void* x, float* master, void* params, int64_t n, float step, void* stream) {
  if (n % 8) return 1;
  muon_apply_kernel<<<stream_grid(n / 8), 256, 0, (cudaStream_t)stream>>>(
      static_cast<const __nv_bfloat16*>(x), master, static_cast<__nv_bfloat16*>(params), n / 8, step);
  return last_launch_rc();
}

int launch_normuon(const void* x, float* buf, int rows, int cols, float beta2, float* vmean,
                   float* factor, void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  normuon_rows_kernel<<<(rows + 7) / 8, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), buf, rows,
                                                      cols, beta2, vmean, factor);
  normuon_scale_kernel<<<1, 1024, 0, st>>>(vmean, factor, rows);
  return last_launch_rc();
}

int launch_muon_apply_rows(const void* x, float* master, void* params, int rows, int cols,
                           float step, const float* factor, void* stream) {
  const int64_t n = int64_t(rows) * cols;
  if (n % 8) return 1;
  muon_apply_rows_kernel<<<stream_grid(n / 8), 256, 0, (cudaStream_t)stream>>>(
      static_cast<const __nv_bfloat16*>(x), master, static_cast<__nv_bfloat16*>(params), n / 8, cols,
      step, factor);
  return last_launch_rc();
}

}  // namespace gpt
