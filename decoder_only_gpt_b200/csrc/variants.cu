// Block variants of the GPT ("ChatGPT'nizi 50 Dolara Nasil Egitirsiniz?",
// section "1. GPT Modeli": the value-embedding (ResFormer) and efficiency-trick
// listings): value embeddings with a per-head gate, per-layer residual
// scaling, smear and backout, forward and backward.  All element-wise or
// row-wise (HBM-bound); every reduction runs on a fixed grid in a fixed
// order, so results are bit-identical from run to run.
//
// T is the storage type of activations and parameters (bf16, or fp32 for the
// fp32 configuration); the residual stream and its gradient are fp32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "device_common.cuh"
#include "gpt_internal.h"

namespace gpt {
namespace {

// fixed grid of the deterministic flat dot products: 8 blocks of 256 threads
// per SM, enough warps in flight to keep HBM busy
constexpr int kRedBlocks = 148 * 8;

__device__ __forceinline__ float sigmoidf_(float z) { return 1.f / (1.f + __expf(-z)); }

// four consecutive elements of T, as one 8- (bf16) or 16-byte (fp32) access
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  *reinterpret_cast<uint2*>(p) =
      make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
}

template <typename T>
__device__ __forceinline__ void store_acc(T* out, float v, int accumulate) {
  if (accumulate) v += to_f(*out);
  *out = from_f<T>(v);
}

// Smear, forward: warp per position t of a sequence of T positions.
//   u = e_t[:24] . w,  sg = sigmoid(u),  x_t = e_t + s sg e_{t-1} (e_{-1} = 0)
template <typename T>
__global__ void smear_fwd_kernel(const float* __restrict__ e, const T* __restrict__ w,
                                 const T* __restrict__ scalars, float* __restrict__ x,
                                 float* __restrict__ sg_out, int64_t N, int Tlen, int d) {
  const int64_t t = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (t >= N) return;
  const float* et = e + t * d;
  float u = lane < kSmearChannels ? et[lane] * to_f(w[lane]) : 0.f;
  u = warp_sum(u);
  const float sg = sigmoidf_(u), g = to_f(scalars[0]) * sg;
  const bool first = t % Tlen == 0;
  const float* ep = et - d;
  for (int c = lane; c < d; c += 32) x[t * d + c] = et[c] + (first ? 0.f : g * ep[c]);
  if (lane == 0) sg_out[t] = sg;
}

// Residual scaling, forward: xprev = x;  x = a x + b x0  (a, b = lam[l, 0..1])
template <typename T>
__global__ void lambda_mix_kernel(float* __restrict__ x, const float* __restrict__ x0,
                                  float* __restrict__ xprev, const T* __restrict__ lam, int64_t n4) {
  const float a = to_f(lam[0]), b = to_f(lam[1]);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(x)[i];
    const float4 z = reinterpret_cast<const float4*>(x0)[i];
    reinterpret_cast<float4*>(xprev)[i] = v;
    reinterpret_cast<float4*>(x)[i] =
        make_float4(a * v.x + b * z.x, a * v.y + b * z.y, a * v.z + b * z.z, a * v.w + b * z.w);
  }
}

// y += mul * (s ? s[0] : 1) * x   (backout forward; the x0 term of the backward)
template <typename T>
__global__ void axpy_kernel(float* __restrict__ y, const float* __restrict__ x, const T* s, float mul,
                            int64_t n4) {
  const float alpha = mul * (s ? to_f(s[0]) : 1.f);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(x)[i];
    float4 o = reinterpret_cast<float4*>(y)[i];
    o.x += alpha * v.x; o.y += alpha * v.y; o.z += alpha * v.z; o.w += alpha * v.w;
    reinterpret_cast<float4*>(y)[i] = o;
  }
}

// Value embedding, forward: warp per (token, key/value head).
//   gz = h_t[:C] . Wg[hk],  v[b, hk, t] += 3 sigmoid(gz) VE[tok_t, hk]
template <typename T>
__global__ void ve_fwd_kernel(const T* __restrict__ h, const T* __restrict__ wg, const T* __restrict__ ve,
                              const int32_t* __restrict__ tok, T* __restrict__ v, int64_t N, int Tlen,
                              int d, int Hkv, int hd, int C, int V) {
  const int64_t item = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (item >= N * Hkv) return;
  const int64_t t = item / Hkv;
  const int hk = int(item % Hkv);
  float gz = 0.f;
  for (int c = lane; c < C; c += 32) gz += to_f(h[t * d + c]) * to_f(wg[hk * C + c]);
  gz = warp_sum(gz);
  const float gate = 3.f * sigmoidf_(gz);
  int id = tok[t];
  id = id < 0 || id >= V ? 0 : id;  // out-of-range ids are reported by the embedding gather
  const T* row = ve + int64_t(id) * Hkv * hd + hk * hd;
  const int64_t b = t / Tlen, tt = t % Tlen;
  T* vr = v + ((b * Hkv + hk) * Tlen + tt) * hd;
  if ((hd & 3) == 0) {
    for (int i = 4 * lane; i < hd; i += 128) {
      const float4 a = load4(vr + i), e = load4(row + i);
      store4(vr + i, make_float4(a.x + gate * e.x, a.y + gate * e.y, a.z + gate * e.z, a.w + gate * e.w));
    }
  } else {
    for (int i = lane; i < hd; i += 32) vr[i] = from_f<T>(to_f(vr[i]) + gate * to_f(row[i]));
  }
}

// Value embedding, backward: warp per (token, key/value head).  dv is the v
// part of the [q | k | v] gradient rows (token-major, ld = q/k/v columns).
//   rows[t, hk] = gate dv   (the table gradient before the scatter by token)
//   dgz[t, hk] = (dv . VE[tok_t, hk]) 3 sigmoid'(gz)
template <typename T>
__global__ void ve_bwd_kernel(const T* __restrict__ dqkv, int64_t ldq, int64_t v_col0,
                              const T* __restrict__ h, const T* __restrict__ wg, const T* __restrict__ ve,
                              const int32_t* __restrict__ tok, float* __restrict__ rows,
                              float* __restrict__ dgz, int64_t N, int d, int Hkv, int hd, int C, int V) {
  const int64_t item = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (item >= N * Hkv) return;
  const int64_t t = item / Hkv;
  const int hk = int(item % Hkv);
  float gz = 0.f;
  for (int c = lane; c < C; c += 32) gz += to_f(h[t * d + c]) * to_f(wg[hk * C + c]);
  gz = warp_sum(gz);
  const float sg = sigmoidf_(gz), gate = 3.f * sg;
  int id = tok[t];
  id = id < 0 || id >= V ? 0 : id;
  const T* row = ve + int64_t(id) * Hkv * hd + hk * hd;
  const T* dv = dqkv + t * ldq + v_col0 + hk * hd;
  float* out = rows + (t * Hkv + hk) * hd;
  float s = 0.f;
  if ((hd & 3) == 0 && (ldq & 3) == 0 && (v_col0 & 3) == 0) {
    for (int i = 4 * lane; i < hd; i += 128) {
      const float4 g = load4(dv + i), e = load4(row + i);
      s += g.x * e.x + g.y * e.y + g.z * e.z + g.w * e.w;
      store4(out + i, make_float4(gate * g.x, gate * g.y, gate * g.z, gate * g.w));
    }
  } else {
    for (int i = lane; i < hd; i += 32) {
      const float g = to_f(dv[i]);
      s += g * to_f(row[i]);
      out[i] = gate * g;
    }
  }
  s = warp_sum(s);
  if (lane == 0) dgz[item] = s * 3.f * sg * (1.f - sg);
}

// dh[t, c] += sum_hk dgz[t, hk] Wg[hk, c]  for c < C (the gate's input)
template <typename T>
__global__ void ve_dh_kernel(T* __restrict__ dh, const float* __restrict__ dgz, const T* __restrict__ wg,
                             int64_t N, int d, int Hkv, int C) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= N * C) return;
  const int64_t t = i / C;
  const int c = int(i % C);
  float s = 0.f;
  for (int hk = 0; hk < Hkv; ++hk) s += dgz[t * Hkv + hk] * to_f(wg[hk * C + c]);
  dh[t * d + c] = from_f<T>(to_f(dh[t * d + c]) + s);
}

// out[i, j] (+)= scale * sum_t a[t * lda + i] * b[t * ldb + j]: one block per
// (i, j), threads over t in a fixed stride, then a fixed tree.
template <typename TB, typename TO>
__global__ void coldot_kernel(const float* __restrict__ a, int64_t lda, const TB* __restrict__ b,
                              int64_t ldb, int nb, int64_t N, float scale, TO* __restrict__ out,
                              int accumulate) {
  const int i = int(blockIdx.x) / nb, j = int(blockIdx.x) % nb;
  float s = 0.f;
  for (int64_t t = threadIdx.x; t < N; t += blockDim.x) s += a[t * lda + i] * to_f(b[t * ldb + j]);
  __shared__ float red[32];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = warp_sum(threadIdx.x < blockDim.x / 32 ? red[threadIdx.x] : 0.f);
    if (threadIdx.x == 0) store_acc(out + blockIdx.x, scale * s, accumulate);
  }
}

// Per-block partial sums of x . y over n elements (fixed grid kRedBlocks).
__global__ void dot_partial_kernel(const float* __restrict__ x, const float* __restrict__ y, int64_t n4,
                                   float* __restrict__ partial) {
  float s = 0.f;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float4 u = reinterpret_cast<const float4*>(x)[i], v = reinterpret_cast<const float4*>(y)[i];
    s += u.x * v.x + u.y * v.y + u.z * v.z + u.w * v.w;
  }
  __shared__ float red[32];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = warp_sum(threadIdx.x < blockDim.x / 32 ? red[threadIdx.x] : 0.f);
    if (threadIdx.x == 0) partial[blockIdx.x] = s;
  }
}

// out[k] (+)= scale * sum of partial[k * nb .. (k+1) * nb), in order, k < nout
template <typename T>
__global__ void dot_finalize_kernel(const float* __restrict__ partial, int nb, int nout, float scale,
                                    T* __restrict__ out, int accumulate) {
  const int k = threadIdx.x / 32, lane = threadIdx.x & 31;
  if (k >= nout) return;
  float s = 0.f;
  for (int i = lane; i < nb; i += 32) s += partial[k * nb + i];
  s = warp_sum(s);
  if (lane == 0) store_acc(out + k, scale * s, accumulate);
}

// Residual backward at a layer's entry, over the fp32 stream gradient dx:
//   backout (bo): dx += -beta dxf            (x_b is this layer's input)
//   scaling (lam): partials of dx . xprev and dx . x0 (d lam[l, 0..1]),
//                  dx0 += b dx,  dx = a dx
// and the storage copy dxs = T(dx) that the next GEMMs read.
template <typename T>
__global__ void resid_bwd_kernel(float* __restrict__ dx, T* __restrict__ dxs, const float* __restrict__ dxf,
                                 const T* __restrict__ scalars, const float* __restrict__ xprev,
                                 const float* __restrict__ x0, float* __restrict__ dx0,
                                 const T* __restrict__ lam, int64_t n4, float* __restrict__ partial) {
  const float beta = dxf ? to_f(scalars[1]) : 0.f;
  const float a = lam ? to_f(lam[0]) : 1.f, b = lam ? to_f(lam[1]) : 0.f;
  float sa = 0.f, sb = 0.f;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += int64_t(gridDim.x) * blockDim.x) {
    float4 g = reinterpret_cast<float4*>(dx)[i];
    if (dxf) {
      const float4 f = reinterpret_cast<const float4*>(dxf)[i];
      g.x -= beta * f.x; g.y -= beta * f.y; g.z -= beta * f.z; g.w -= beta * f.w;
    }
    if (lam) {
      const float4 p = reinterpret_cast<const float4*>(xprev)[i];
      const float4 z = reinterpret_cast<const float4*>(x0)[i];
      sa += g.x * p.x + g.y * p.y + g.z * p.z + g.w * p.w;
      sb += g.x * z.x + g.y * z.y + g.z * z.z + g.w * z.w;
      float4 acc = reinterpret_cast<float4*>(dx0)[i];
      acc.x += b * g.x; acc.y += b * g.y; acc.z += b * g.z; acc.w += b * g.w;
      reinterpret_cast<float4*>(dx0)[i] = acc;
      g.x *= a; g.y *= a; g.z *= a; g.w *= a;
    }
    reinterpret_cast<float4*>(dx)[i] = g;
    store4(dxs + 4 * i, g);
  }
  if (!lam) return;
  __shared__ float red[2][32];
  sa = warp_sum(sa);
  sb = warp_sum(sb);
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x / 32] = sa;
    red[1][threadIdx.x / 32] = sb;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const bool in = threadIdx.x < blockDim.x / 32;
    sa = warp_sum(in ? red[0][threadIdx.x] : 0.f);
    sb = warp_sum(in ? red[1][threadIdx.x] : 0.f);
    if (threadIdx.x == 0) {
      partial[blockIdx.x] = sa;
      partial[gridDim.x + blockIdx.x] = sb;
    }
  }
}

// Smear, backward, step 1: warp per position.  dg = dx_t . e_{t-1};
// du = dg s sg (1 - sg)
template <typename T>
__global__ void smear_bwd1_kernel(const float* __restrict__ dx, const float* __restrict__ e,
                                  const float* __restrict__ sg, const T* __restrict__ scalars,
                                  float* __restrict__ dg_out, float* __restrict__ du_out, int64_t N,
                                  int Tlen, int d) {
  const float s = to_f(scalars[0]);
  const int64_t t = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (t >= N) return;
  float dg = 0.f;
  if (t % Tlen != 0)
    for (int c = lane; c < d; c += 32) dg += dx[t * d + c] * e[(t - 1) * d + c];
  dg = warp_sum(dg);
  if (lane == 0) {
    dg_out[t] = dg;
    du_out[t] = dg * s * sg[t] * (1.f - sg[t]);
  }
}

// Smear, backward, step 2: de_t = dx_t + s sg_{t+1} dx_{t+1} (same sequence)
// + du_t w on the gate's 24 channels, written over e.
template <typename T>
__global__ void smear_bwd2_kernel(const float* __restrict__ dx, const float* __restrict__ sg,
                                  const float* __restrict__ du, const T* __restrict__ w,
                                  const T* __restrict__ scalars, float* __restrict__ de, int64_t N,
                                  int Tlen, int d) {
  const float s = to_f(scalars[0]);
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= N * d) return;
  const int64_t t = i / d;
  const int c = int(i % d);
  float v = dx[i];
  if (t % Tlen != Tlen - 1 && t + 1 < N) v += s * sg[t + 1] * dx[i + d];
  if (c < kSmearChannels) v += du[t] * to_f(w[c]);
  de[i] = v;
}

int grid_for(int64_t n, int per_block) {
  const int64_t g = (n + per_block - 1) / per_block;
  return int(g < 1 ? 1 : g);
}
int stream_grid4(int64_t n4) {
  const int64_t want = (n4 + 255) / 256;
  return int(want < 148 * 8 ? (want > 0 ? want : 1) : 148 * 8);
}

}  // namespace

// ---- launchers ------------------------------------------------------------
// (T by the config's dtype; sizes in elements; every pointer device memory)

#define VAR_DISPATCH(c, CALL)                                         \
  do {                                                                \
    if ((c).dtype == GPT_BF16) { using T = __nv_bfloat16; CALL; }     \
    else { using T = float; CALL; }                                   \
  } while (0)

int launch_smear_fwd(const gpt_config& c, const float* e, const void* w, const void* scalars, float* x,
                     float* sg, void* stream) {
  const int64_t N = int64_t(c.batch) * c.seq_len;
  VAR_DISPATCH(c, (smear_fwd_kernel<T><<<grid_for(N, 8), 256, 0, (cudaStream_t)stream>>>(
                      e, static_cast<const T*>(w), static_cast<const T*>(scalars), x, sg, N, c.seq_len,
                      c.d_model)));
  return last_launch_rc();
}

int launch_lambda_mix(const gpt_config& c, float* x, const float* x0, float* xprev, const void* lam,
                      void* stream) {
  const int64_t n4 = int64_t(c.batch) * c.seq_len * c.d_model / 4;
  VAR_DISPATCH(c, (lambda_mix_kernel<T><<<stream_grid4(n4), 256, 0, (cudaStream_t)stream>>>(
                      x, x0, xprev, static_cast<const T*>(lam), n4)));
  return last_launch_rc();
}

int launch_axpy(const gpt_config& c, float* y, const float* x, const void* s, float mul, void* stream) {
  const int64_t n4 = int64_t(c.batch) * c.seq_len * c.d_model / 4;
  VAR_DISPATCH(c, (axpy_kernel<T><<<stream_grid4(n4), 256, 0, (cudaStream_t)stream>>>(
                      y, x, static_cast<const T*>(s), mul, n4)));
  return last_launch_rc();
}

int launch_ve_fwd(const gpt_config& c, const void* h, const void* wg, const void* ve, const int32_t* tok,
                  void* v, void* stream) {
  const int64_t N = int64_t(c.batch) * c.seq_len;
  VAR_DISPATCH(c, (ve_fwd_kernel<T><<<grid_for(N * c.n_kv_head, 8), 256, 0, (cudaStream_t)stream>>>(
                      static_cast<const T*>(h), static_cast<const T*>(wg), static_cast<const T*>(ve), tok,
                      static_cast<T*>(v), N, c.seq_len, c.d_model, c.n_kv_head, c.head_dim,
                      c.ve_gate_channels, c.vocab)));
  return last_launch_rc();
}

int launch_ve_bwd(const gpt_config& c, const void* dqkv, const void* h, const void* wg, const void* ve,
                  const int32_t* tok, float* rows, float* dgz, void* d_wg, int accumulate, void* stream) {
  const int64_t N = int64_t(c.batch) * c.seq_len;
  const int64_t ldq = qkv_cols(c), v_col0 = int64_t(c.d_model) + int64_t(c.n_kv_head) * c.head_dim;
  cudaStream_t st = (cudaStream_t)stream;
  VAR_DISPATCH(c, (ve_bwd_kernel<T><<<grid_for(N * c.n_kv_head, 8), 256, 0, st>>>(
                      static_cast<const T*>(dqkv), ldq, v_col0, static_cast<const T*>(h),
                      static_cast<const T*>(wg), static_cast<const T*>(ve), tok, rows, dgz, N, c.d_model,
                      c.n_kv_head, c.head_dim, c.ve_gate_channels, c.vocab)));
  if (last_launch_rc()) return 1;
  // d Wg[hk, c] = sum_t dgz[t, hk] h[t, c]
  VAR_DISPATCH(c, (coldot_kernel<T, T><<<c.n_kv_head * c.ve_gate_channels, 256, 0, st>>>(
                      dgz, c.n_kv_head, static_cast<const T*>(h), c.d_model, c.ve_gate_channels, N, 1.f,
                      static_cast<T*>(d_wg), accumulate)));
  return last_launch_rc();
}

int launch_ve_dh(const gpt_config& c, void* dh, const float* dgz, const void* wg, void* stream) {
  const int64_t N = int64_t(c.batch) * c.seq_len;
  VAR_DISPATCH(c, (ve_dh_kernel<T><<<grid_for(N * c.ve_gate_channels, 256), 256, 0, (cudaStream_t)stream>>>(
                      static_cast<T*>(dh), dgz, static_cast<const T*>(wg), N, c.d_model, c.n_kv_head,
                      c.ve_gate_channels)));
  return last_launch_rc();
}

int launch_resid_bwd(const gpt_config& c, float* dx, void* dxs, const float* dxf, const void* scalars,
                     const float* xprev, const float* x0, float* dx0, const void* lam, float* partial,
                     void* d_lam, int accumulate, void* stream) {
  const int64_t n4 = int64_t(c.batch) * c.seq_len * c.d_model / 4;
  cudaStream_t st = (cudaStream_t)stream;
  VAR_DISPATCH(c, (resid_bwd_kernel<T><<<kRedBlocks, 256, 0, st>>>(
                      dx, static_cast<T*>(dxs), dxf, static_cast<const T*>(scalars), xprev, x0, dx0,
                      static_cast<const T*>(lam), n4, partial)));
  if (last_launch_rc()) return 1;
  if (lam)
    VAR_DISPATCH(c, (dot_finalize_kernel<T><<<1, 64, 0, st>>>(partial, kRedBlocks, 2, 1.f,
                                                              static_cast<T*>(d_lam), accumulate)));
  return last_launch_rc();
}

int launch_dot(const gpt_config& c, const float* x, const float* y, float scale, float* partial,
               void* out, int accumulate, void* stream) {
  const int64_t n4 = int64_t(c.batch) * c.seq_len * c.d_model / 4;
  cudaStream_t st = (cudaStream_t)stream;
  dot_partial_kernel<<<kRedBlocks, 256, 0, st>>>(x, y, n4, partial);
  if (last_launch_rc()) return 1;
  VAR_DISPATCH(c, (dot_finalize_kernel<T><<<1, 32, 0, st>>>(partial, kRedBlocks, 1, scale,
                                                            static_cast<T*>(out), accumulate)));
  return last_launch_rc();
}

int launch_smear_bwd(const gpt_config& c, const float* dx, float* e, const float* sg, float* dg,
                     float* du, const void* w, const void* scalars, void* d_w, void* d_scalars,
                     int accumulate, void* stream) {
  const int64_t N = int64_t(c.batch) * c.seq_len;
  const int d = c.d_model;
  cudaStream_t st = (cudaStream_t)stream;
  VAR_DISPATCH(c, (smear_bwd1_kernel<T><<<grid_for(N, 8), 256, 0, st>>>(
                      dx, e, sg, static_cast<const T*>(scalars), dg, du, N, c.seq_len, d)));
  if (last_launch_rc()) return 1;
  // d w[c] = sum_t du_t e_t[c] (before e is overwritten); d s = sum_t dg_t sg_t
  VAR_DISPATCH(c, (coldot_kernel<float, T><<<kSmearChannels, 256, 0, st>>>(
                      du, 1, e, d, kSmearChannels, N, 1.f, static_cast<T*>(d_w), accumulate)));
  VAR_DISPATCH(c, (coldot_kernel<float, T><<<1, 256, 0, st>>>(dg, 1, sg, 1, 1, N, 1.f,
                                                               static_cast<T*>(d_scalars), accumulate)));
  VAR_DISPATCH(c, (smear_bwd2_kernel<T><<<grid_for(N * d, 256), 256, 0, st>>>(
                      dx, sg, du, static_cast<const T*>(w), static_cast<const T*>(scalars), e, N,
                      c.seq_len, d)));
  return last_launch_rc();
}

int variant_red_floats() { return 2 * kRedBlocks + 64; }

}  // namespace gpt
