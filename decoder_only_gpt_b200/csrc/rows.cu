// Row-wise kernels of the step: token-embedding gather fused with the first
// RMSNorm, parameter-free RMSNorm forward / backward, RoPE + QK-norm of the
// projected q/k (with the head-major scatter of q, k, v), the cross-entropy
// merge of per-tile partial statistics and the deterministic loss mean.
//
// All are HBM-bound: one warp per row, lane-strided (coalesced) accesses,
// fp32 statistics, warp-shuffle reductions.
#include <math.h>

#include "device_common.cuh"

namespace gpt {

// ---------------------------------------------------------------------------
// RoPE table: angle(t, i) = t * base^(-2i/hd), evaluated in fp64, stored fp32,
// both position-major [T, hd/2] and pair-major [hd/2, T] (the QKV epilogue's
// threads hold consecutive positions, so a pair-major row is one coalesced load)
// ---------------------------------------------------------------------------
__global__ void rope_table_kernel(float* cos_t, float* sin_t, float* cos_tr, float* sin_tr, int T, int half,
                                  double base, int hd) {
  int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= T * half) return;
  int t = idx / half, i = idx % half;
  double theta = pow(base, -2.0 * double(i) / double(hd));
  double s, c;
  sincos(double(t) * theta, &s, &c);
  cos_t[idx] = float(c);
  sin_t[idx] = float(s);
  cos_tr[int64_t(i) * T + t] = float(c);
  sin_tr[int64_t(i) * T + t] = float(s);
}

int launch_rope_table(const gpt_config& c, float* cos_t, float* sin_t, float* cos_tr, float* sin_tr,
                      void* stream) {
  int half = c.head_dim / 2, n = c.seq_len * half;
  rope_table_kernel<<<ceil_div(n, 256), 256, 0, (cudaStream_t)stream>>>(
      cos_t, sin_t, cos_tr, sin_tr, c.seq_len, half, double(c.rope_base), c.head_dim);
  return last_launch_rc();
}

// ---------------------------------------------------------------------------
// x = wte[token] (exact upcast to fp32), h = rms(x), r = 1/sqrt(mean(x^2)+eps)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void embed_norm_kernel(const int32_t* __restrict__ tok, const T* __restrict__ wte,
                                  float* __restrict__ x, T* __restrict__ h, float* __restrict__ r,
                                  int64_t N, int d, int V, float eps, int32_t* status) {
  int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  int lane = threadIdx.x & 31;
  if (row >= N) return;
  int id = tok[row];
  if (id < 0 || id >= V) {
    if (lane == 0) record_status(status, GPT_EDATA, K_EMBED, row);
    id = 0;
  }
  const T* src = wte + int64_t(id) * d;
  float* xr = x + row * d;
  float ss = 0.f;
  for (int i = lane; i < d; i += 32) {
    float v = to_f(src[i]);
    xr[i] = v;
    ss += v * v;
  }
  ss = warp_sum(ss);
  float rr = rsqrtf(ss / float(d) + eps);
  T* hr = h + row * d;
  for (int i = lane; i < d; i += 32) hr[i] = from_f<T>(to_f(src[i]) * rr);
  if (lane == 0) r[row] = rr;
}

int launch_embed_norm(const gpt_config& c, const int32_t* tok, const void* wte, float* x,
                      void* h, float* r, int32_t* status, void* stream) {
  int64_t N = int64_t(c.batch) * c.seq_len;
  dim3 grid(ceil_div(N, 8));
  if (c.dtype == GPT_BF16)
    embed_norm_kernel<__nv_bfloat16><<<grid, 256, 0, (cudaStream_t)stream>>>(
        tok, (const __nv_bfloat16*)wte, x, (__nv_bfloat16*)h, r, N, c.d_model, c.vocab,
        c.norm_eps, status);
  else
    embed_norm_kernel<float><<<grid, 256, 0, (cudaStream_t)stream>>>(
        tok, (const float*)wte, x, (float*)h, r, N, c.d_model, c.vocab, c.norm_eps, status);
  return last_launch_rc();
}

// ---------------------------------------------------------------------------
// RMSNorm forward of the fp32 residual stream.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void rms_fwd_kernel(const float* __restrict__ x, T* __restrict__ h,
                               float* __restrict__ r, int64_t N, int d, float eps) {
  int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  int lane = threadIdx.x & 31;
  if (row >= N) return;
  const float* xr = x + row * d;
  float ss = 0.f;
  if ((d & 3) == 0) {
    const float4* x4 = reinterpret_cast<const float4*>(xr);
    for (int i = lane; i < d / 4; i += 32) {
      float4 v = x4[i];
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
  } else {
    for (int i = lane; i < d; i += 32) ss += xr[i] * xr[i];
  }
  ss = warp_sum(ss);
  float rr = rsqrtf(ss / float(d) + eps);
  T* hr = h + row * d;
  for (int i = lane; i < d; i += 32) hr[i] = from_f<T>(xr[i] * rr);
  if (lane == 0) r[row] = rr;
}

// bf16 output, d % 8 == 0 and d <= 8 * 32 * kMaxVec: 16-byte accesses, the row in registers.
constexpr int kMaxVec = 8;  // 8-element groups per lane: d <= 2048

__device__ __forceinline__ uint32_t pk_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 up_bf16(uint32_t u) {
  return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u));
}
__device__ __forceinline__ void up8(const uint4& u, float (&f)[8]) {
  float2 a = up_bf16(u.x), b = up_bf16(u.y), c = up_bf16(u.z), d = up_bf16(u.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

__global__ void rms_fwd_bf16_vec(const float* __restrict__ x, __nv_bfloat16* __restrict__ h,
                                 float* __restrict__ r, int64_t N, int d, float eps) {
  const int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const int groups = d / 8;
  const float4* xr = reinterpret_cast<const float4*>(x + row * d);
  float4 va[kMaxVec], vb[kMaxVec];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < kMaxVec; ++k) {
    const int gi = lane + 32 * k;
    if (gi < groups) {
      va[k] = xr[2 * gi];
      vb[k] = xr[2 * gi + 1];
      ss += va[k].x * va[k].x + va[k].y * va[k].y + va[k].z * va[k].z + va[k].w * va[k].w +
            vb[k].x * vb[k].x + vb[k].y * vb[k].y + vb[k].z * vb[k].z + vb[k].w * vb[k].w;
    }
  }
  ss = warp_sum(ss);
  const float rr = rsqrtf(ss / float(d) + eps);
  uint4* hr = reinterpret_cast<uint4*>(h + row * d);
#pragma unroll
  for (int k = 0; k < kMaxVec; ++k) {
    const int gi = lane + 32 * k;
    if (gi < groups)
      hr[gi] = make_uint4(pk_bf16(va[k].x * rr, va[k].y * rr), pk_bf16(va[k].z * rr, va[k].w * rr),
                          pk_bf16(vb[k].x * rr, vb[k].y * rr), pk_bf16(vb[k].z * rr, vb[k].w * rr));
  }
  if (lane == 0) r[row] = rr;
}

int launch_rms_fwd(const gpt_config& c, const float* x, void* h, float* r, void* stream) {
  int64_t N = int64_t(c.batch) * c.seq_len;
  dim3 grid(ceil_div(N, 8));
  if (c.dtype == GPT_BF16 && c.d_model % 8 == 0 && c.d_model <= 8 * 32 * kMaxVec)
    rms_fwd_bf16_vec<<<grid, 256, 0, (cudaStream_t)stream>>>(x, (__nv_bfloat16*)h, r, N,
                                                            c.d_model, c.norm_eps);
  else if (c.dtype == GPT_BF16)
    rms_fwd_kernel<__nv_bfloat16><<<grid, 256, 0, (cudaStream_t)stream>>>(
        x, (__nv_bfloat16*)h, r, N, c.d_model, c.norm_eps);
  else
    rms_fwd_kernel<float><<<grid, 256, 0, (cudaStream_t)stream>>>(x, (float*)h, r, N,
                                                                  c.d_model, c.norm_eps);
  return last_launch_rc();
}

// ---------------------------------------------------------------------------
// RMSNorm backward into the fp32 residual gradient:
//   dx (+)= r * (dh - h * mean(dh * h));  dxs = storage copy of dx (GEMM operand)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void rms_bwd_kernel(const T* __restrict__ dh, const T* __restrict__ h,
                               const float* __restrict__ r, float* __restrict__ dx,
                               T* __restrict__ dxs, int64_t N, int d, int accumulate) {
  int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  int lane = threadIdx.x & 31;
  if (row >= N) return;
  const T* dr = dh + row * d;
  const T* hr = h + row * d;
  float s = 0.f;
  for (int i = lane; i < d; i += 32) s += to_f(dr[i]) * to_f(hr[i]);
  s = warp_sum(s) / float(d);
  float rr = r[row];
  float* xr = dx + row * d;
  T* sr = dxs + row * d;
  for (int i = lane; i < d; i += 32) {
    float g = rr * (to_f(dr[i]) - to_f(hr[i]) * s);
    if (accumulate) g += xr[i];
    xr[i] = g;
    sr[i] = from_f<T>(g);
  }
}

// bf16, d % 8 == 0, d <= 8 * 32 * KV: a row's dh and h loads are issued
// before the row reduction, so their latencies overlap; the fp32 dx it
// accumulates into is read after it (fewer live registers, more warps per SM
// to cover the latency); KV = the 8-element groups per lane, sized to d.
template <int KV>
__global__ void rms_bwd_bf16_vec(const __nv_bfloat16* __restrict__ dh,
                                 const __nv_bfloat16* __restrict__ h, const float* __restrict__ r,
                                 float* __restrict__ dx, __nv_bfloat16* __restrict__ dxs,
                                 int64_t N, int d, int accumulate) {
  const int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const int groups = d / 8;
  const uint4* dr = reinterpret_cast<const uint4*>(dh + row * d);
  const uint4* hr = reinterpret_cast<const uint4*>(h + row * d);
  float4* xr = reinterpret_cast<float4*>(dx + row * d);
  uint4 gd[KV], gh[KV];
#pragma unroll
  for (int k = 0; k < KV; ++k) {
    const int gi = lane + 32 * k;
    if (gi < groups) {
      gd[k] = dr[gi];
      gh[k] = hr[gi];
    }
  }
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < KV; ++k) {
    const int gi = lane + 32 * k;
    if (gi < groups) {
      float fa[8], fb[8];
      up8(gd[k], fa);
      up8(gh[k], fb);
#pragma unroll
      for (int e = 0; e < 8; ++e) s += fa[e] * fb[e];
    }
  }
  s = warp_sum(s) / float(d);
  const float rr = r[row];
  uint4* sr = reinterpret_cast<uint4*>(dxs + row * d);
#pragma unroll
  for (int k = 0; k < KV; ++k) {
    const int gi = lane + 32 * k;
    if (gi < groups) {
      float fa[8], fb[8], g[8];
      up8(gd[k], fa);
      up8(gh[k], fb);
#pragma unroll
      for (int e = 0; e < 8; ++e) g[e] = rr * (fa[e] - fb[e] * s);
      if (accumulate) {
        const float4 p0 = xr[2 * gi], p1 = xr[2 * gi + 1];
        g[0] += p0.x; g[1] += p0.y; g[2] += p0.z; g[3] += p0.w;
        g[4] += p1.x; g[5] += p1.y; g[6] += p1.z; g[7] += p1.w;
      }
      xr[2 * gi] = make_float4(g[0], g[1], g[2], g[3]);
      xr[2 * gi + 1] = make_float4(g[4], g[5], g[6], g[7]);
      sr[gi] = make_uint4(pk_bf16(g[0], g[1]), pk_bf16(g[2], g[3]), pk_bf16(g[4], g[5]),
                          pk_bf16(g[6], g[7]));
    }
  }
}

int launch_rms_bwd(const gpt_config& c, const void* dh, const void* h, const float* r,
                   float* dx, void* dxs, int accumulate, void* stream) {
  int64_t N = int64_t(c.batch) * c.seq_len;
  dim3 grid(ceil_div(N, 8));
  if (c.dtype == GPT_BF16 && c.d_model % 8 == 0 && c.d_model <= 8 * 32 * kMaxVec) {
    const int kv = (c.d_model / 8 + 31) / 32;  // 8-element groups per lane
    auto args = [&](auto kern) {
      kern<<<grid, 256, 0, (cudaStream_t)stream>>>((const __nv_bfloat16*)dh, (const __nv_bfloat16*)h, r,
                                                   dx, (__nv_bfloat16*)dxs, N, c.d_model, accumulate);
    };
    switch (kv) {
      case 1: args(rms_bwd_bf16_vec<1>); break;
      case 2: args(rms_bwd_bf16_vec<2>); break;
      case 3: args(rms_bwd_bf16_vec<3>); break;
      case 4: args(rms_bwd_bf16_vec<4>); break;
      case 5: args(rms_bwd_bf16_vec<5>); break;
      case 6: args(rms_bwd_bf16_vec<6>); break;
      case 7: args(rms_bwd_bf16_vec<7>); break;
      default: args(rms_bwd_bf16_vec<8>); break;
    }
  } else if (c.dtype == GPT_BF16)
    rms_bwd_kernel<__nv_bfloat16><<<grid, 256, 0, (cudaStream_t)stream>>>(
        (const __nv_bfloat16*)dh, (const __nv_bfloat16*)h, r, dx, (__nv_bfloat16*)dxs, N,
        c.d_model, accumulate);
  else
    rms_bwd_kernel<float><<<grid, 256, 0, (cudaStream_t)stream>>>(
        (const float*)dh, (const float*)h, r, dx, (float*)dxs, N, c.d_model, accumulate);
  return last_launch_rc();
}

// ---------------------------------------------------------------------------
// q, k <- rms_head(RoPE(q, k)); scatter q, k, v from [N, Q] rows (n_head q
// heads, then Hkv k heads and Hkv v heads) to [B, heads, T, hd].  One warp per
// (token, query head); the warps of heads below Hkv also handle that k and v
// head.  A lane handles rotation pairs (i, i + hd/2).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void qkv_post_kernel(const T* __restrict__ raw, const float* __restrict__ cos_t,
                                const float* __restrict__ sin_t, T* __restrict__ q,
                                T* __restrict__ k, T* __restrict__ v, float* __restrict__ rq,
                                float* __restrict__ rk, int64_t N, int Tn, int H, int Hkv, int hd,
                                float eps, int qk_norm) {
  int64_t w = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  int lane = threadIdx.x & 31;
  if (w >= N * H) return;
  int64_t n = w / H;
  int hh = int(w % H);
  int64_t b = n / Tn;
  int t = int(n % Tn);
  const int d = H * hd, half = hd / 2, Q = d + 2 * Hkv * hd;
  for (int part = 0; part < 2; ++part) {
    if (part == 1 && hh >= Hkv) break;
    const int nh = part == 0 ? H : Hkv;
    const int64_t dst = ((b * nh + hh) * Tn + t) * hd;
    const int64_t ridx = (b * nh + hh) * Tn + t;
    const T* src = raw + n * Q + (part == 0 ? 0 : d) + hh * hd;
    T* out = part == 0 ? q : k;
    float a0[4], b0[4];
    float ss = 0.f;
    int cnt = 0;
    for (int i = lane; i < half; i += 32, ++cnt) {
      float x1 = to_f(src[i]), x2 = to_f(src[i + half]);
      float cs = cos_t[t * half + i], sn = sin_t[t * half + i];
      a0[cnt] = x1 * cs - x2 * sn;
      b0[cnt] = x1 * sn + x2 * cs;
      ss += a0[cnt] * a0[cnt] + b0[cnt] * b0[cnt];
    }
    ss = warp_sum(ss);
    float rr = qk_norm ? rsqrtf(ss / float(hd) + eps) : 1.f;
    cnt = 0;
    for (int i = lane; i < half; i += 32, ++cnt) {
      out[dst + i] = from_f<T>(a0[cnt] * rr);
      out[dst + i + half] = from_f<T>(b0[cnt] * rr);
    }
    if (lane == 0) (part == 0 ? rq : rk)[ridx] = rr;
  }
  if (hh >= Hkv) return;
  const T* vs = raw + n * Q + d + Hkv * hd + hh * hd;
  const int64_t vdst = ((b * Hkv + hh) * Tn + t) * hd;
  for (int i = lane; i < hd; i += 32) v[vdst + i] = vs[i];
}

int launch_qkv_post(const gpt_config& c, const void* raw, const float* cos_t,
                    const float* sin_t, void* q, void* k, void* v, float* rq, float* rk,
                    void* stream) {
  int64_t N = int64_t(c.batch) * c.seq_len;
  int64_t warps = N * c.n_head;
  dim3 grid(ceil_div(warps, 8));
  if (c.dtype == GPT_BF16)
    qkv_post_kernel<__nv_bfloat16><<<grid, 256, 0, (cudaStream_t)stream>>>(
        (const __nv_bfloat16*)raw, cos_t, sin_t, (__nv_bfloat16*)q, (__nv_bfloat16*)k,
        (__nv_bfloat16*)v, rq, rk, N, c.seq_len, c.n_head, c.n_kv_head, c.head_dim, c.norm_eps,
        c.qk_norm);
  else
    qkv_post_kernel<float><<<grid, 256, 0, (cudaStream_t)stream>>>(
        (const float*)raw, cos_t, sin_t, (float*)q, (float*)k, (float*)v, rq, rk, N,
        c.seq_len, c.n_head, c.n_kv_head, c.head_dim, c.norm_eps, c.qk_norm);
  return last_launch_rc();
}

// ---------------------------------------------------------------------------
// Cross-entropy merge: lse = M + log(sum_j s_j exp(m_j - M)) over the per-tile
// partials (m_j, s_j) of one row; loss = lse - z[target].
// ---------------------------------------------------------------------------
__global__ void ce_merge_kernel(const float* __restrict__ pmax, const float* __restrict__ psum,
                                int n_part, const float* __restrict__ tgt_logit,
                                const int32_t* __restrict__ tgt, float* __restrict__ lse,
                                float* __restrict__ tok_loss, int64_t N, int V,
                                int32_t* status) {
  int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  int lane = threadIdx.x & 31;
  if (row >= N) return;
  const float* pm = pmax + row * n_part;
  const float* ps = psum + row * n_part;
  float m = -INFINITY;
  for (int j = lane; j < n_part; j += 32) m = fmaxf(m, pm[j]);
  m = warp_max(m);
  float s = 0.f;
  for (int j = lane; j < n_part; j += 32) s += ps[j] * __expf(pm[j] - m);
  s = warp_sum(s);
  if (lane == 0) {
    float l = m + logf(s);
    lse[row] = l;
    int y = tgt[row];
    if (y < 0 || y >= V) {
      record_status(status, GPT_EDATA, K_CE_MERGE, row);
      tok_loss[row] = 0.f;
    } else {
      tok_loss[row] = l - tgt_logit[row];
    }
  }
}

int launch_ce_merge(const gpt_config& c, const float* pmax, const float* psum, int n_part,
                    const float* tgt_logit, const int32_t* tgt, float* lse, float* tok_loss,
                    int32_t* status, void* stream) {
  int64_t N = int64_t(c.batch) * c.seq_len;
  ce_merge_kernel<<<ceil_div(N, 8), 256, 0, (cudaStream_t)stream>>>(
      pmax, psum, n_part, tgt_logit, tgt, lse, tok_loss, N, c.vocab, status);
  return last_launch_rc();
}

// ---------------------------------------------------------------------------
// loss = (1/N) sum_n tok_loss[n], fp64 partial sums in a fixed order.
// ---------------------------------------------------------------------------
__global__ void loss_mean_kernel(const float* __restrict__ tok_loss, float* __restrict__ loss,
                                 float* __restrict__ user_tok_loss, int64_t N,
                                 int32_t* status) {
  __shared__ double part[32];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < N; i += blockDim.x) {
    float v = tok_loss[i];
    s += double(v);
    if (user_tok_loss) user_tok_loss[i] = v;
  }
  s = warp_sum_d(s);
  int w = threadIdx.x / 32, lane = threadIdx.x & 31;
  if (lane == 0) part[w] = s;
  __syncthreads();
  if (w == 0) {
    double t = lane < int(blockDim.x / 32) ? part[lane] : 0.0;
    t = warp_sum_d(t);
    if (lane == 0) {
      float l = float(t / double(N));
      *loss = l;
      if (!isfinite(l)) record_status(status, GPT_ENONFINITE, K_LOSS, -1);
    }
  }
}

int launch_loss_mean(const gpt_config& c, const float* tok_loss, float* loss,
                     float* user_tok_loss, int32_t* status, void* stream) {
  int64_t N = int64_t(c.batch) * c.seq_len;
  loss_mean_kernel<<<1, 1024, 0, (cudaStream_t)stream>>>(tok_loss, loss, user_tok_loss, N,
                                                         status);
  return last_launch_rc();
}

}  // namespace gpt
