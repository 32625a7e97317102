// Causal attention, forward and backward, on CUDA cores (one warp per query or
// key row, scores of the row staged in shared memory).
//
// q: [B, H, T, hd], k, v: [B, Hkv, T, hd] (q, k after RoPE and QK-norm; query
// head h reads key/value head h / (H/Hkv)); o, dO: [B*T, H*hd]; lse: [B, H, T]
// row logsumexp of the scaled scores; dqkv: [B*T, (H + 2 Hkv) hd].  Query t
// sees keys j with t - W < j <= t (W = the window span).
//
// Backward, with D_i = dO_i . o_i and P_ij = exp(s_ij - lse_i):
//   dV_j = sum_i P_ij dO_i;  dS_ij = P_ij (dO_i . v_j - D_i);
//   dQ_i = scale sum_j dS_ij k_j;  dK_j = scale sum_i dS_ij q_i.
// dQ and dK are then taken back through the per-head RMSNorm
// (dx = r (dy - y mean(dy y))) and the RoPE rotation (its transpose), and
// written into the [q | k | v] gradient rows.  dQ (warp per query row) and
// dK/dV (warp per key row) are separate kernels, so no sum needs atomics.
#include "device_common.cuh"

namespace gpt {

namespace {
constexpr int kWarps = 4;
constexpr int kMaxHd = 128;
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
    attn_fwd_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  T* __restrict__ o, float* __restrict__ lse, int H, int Hkv, int Tn, int hd,
                  int W, float scale) {
  extern __shared__ float smem[];
  __shared__ float qs[kWarps][kMaxHd];
  const int w = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + w;
  const int bh = blockIdx.y;
  if (t >= Tn) return;
  float* sc = smem + w * Tn;
  const int64_t base = int64_t(bh) * Tn * hd;
  const int64_t kvbase = (int64_t(bh / H) * Hkv + (bh % H) / (H / Hkv)) * Tn * hd;
  const int j0 = max(0, t - W + 1);
  for (int i = lane; i < hd; i += 32) qs[w][i] = to_f(q[base + int64_t(t) * hd + i]);
  __syncwarp();
  float m = -INFINITY;
  for (int j = j0 + lane; j <= t; j += 32) {
    const T* kr = k + kvbase + int64_t(j) * hd;
    float s = 0.f;
    for (int i = 0; i < hd; ++i) s = fmaf(qs[w][i], to_f(kr[i]), s);
    s *= scale;
    sc[j] = s;
    m = fmaxf(m, s);
  }
  m = warp_max(m);
  float l = 0.f;
  for (int j = j0 + lane; j <= t; j += 32) {
    float p = expf(sc[j] - m);
    sc[j] = p;
    l += p;
  }
  l = warp_sum(l);
  __syncwarp();
  const int b = bh / H, h = bh % H;
  const float inv = 1.f / l;
  for (int i = lane; i < hd; i += 32) {
    float acc = 0.f;
    for (int j = j0; j <= t; ++j) acc = fmaf(sc[j], to_f(v[kvbase + int64_t(j) * hd + i]), acc);
    o[(int64_t(b) * Tn + t) * (H * hd) + h * hd + i] = from_f<T>(acc * inv);
  }
  if (lane == 0) lse[int64_t(bh) * Tn + t] = m + logf(l);
}

// Per-head RMSNorm backward then RoPE backward of one row held in shared
// memory (g: gradient w.r.t. the normalised, rotated row; y: that row),
// written to out[0..hd).
template <typename T>
__device__ __forceinline__ void norm_rope_bwd_row(float* g, const float* y, float r, int qk_norm,
                                                  const float* cosr, const float* sinr, int hd,
                                                  int lane, T* out) {
  if (qk_norm) {
    float s = 0.f;
    for (int i = lane; i < hd; i += 32) s += g[i] * y[i];
    s = warp_sum(s) / float(hd);
    __syncwarp();
    for (int i = lane; i < hd; i += 32) g[i] = r * (g[i] - y[i] * s);
    __syncwarp();
  }
  const int half = hd / 2;
  for (int i = lane; i < half; i += 32) {
    float da = g[i], db = g[i + half], c = cosr[i], s = sinr[i];
    out[i] = from_f<T>(da * c + db * s);
    out[i + half] = from_f<T>(-da * s + db * c);
  }
  __syncwarp();
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
    attn_bwd_dq_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const T* __restrict__ o, const T* __restrict__ dO,
                     const float* __restrict__ lse, const float* __restrict__ rq,
                     const float* __restrict__ cos_t, const float* __restrict__ sin_t,
                     float* __restrict__ Dbuf, T* __restrict__ dqkv, int H, int Hkv, int Tn,
                     int hd, int W, float scale, int qk_norm) {
  extern __shared__ float smem[];
  __shared__ float qs[kWarps][kMaxHd], dos[kWarps][kMaxHd], gs[kWarps][kMaxHd];
  const int w = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + w;
  const int bh = blockIdx.y;
  if (t >= Tn) return;
  const int b = bh / H, h = bh % H, d = H * hd, Q = d + 2 * Hkv * hd;
  float* ds = smem + w * Tn;
  const int64_t base = int64_t(bh) * Tn * hd;
  const int64_t kvbase = (int64_t(b) * Hkv + h / (H / Hkv)) * Tn * hd;
  const int j0 = max(0, t - W + 1);
  const int64_t n = int64_t(b) * Tn + t;
  float D = 0.f;
  for (int i = lane; i < hd; i += 32) {
    float g = to_f(dO[n * d + h * hd + i]);
    dos[w][i] = g;
    D += g * to_f(o[n * d + h * hd + i]);
    qs[w][i] = to_f(q[base + int64_t(t) * hd + i]);
  }
  D = warp_sum(D);
  __syncwarp();
  const float L = lse[int64_t(bh) * Tn + t];
  for (int j = j0 + lane; j <= t; j += 32) {
    const T* kr = k + kvbase + int64_t(j) * hd;
    const T* vr = v + kvbase + int64_t(j) * hd;
    float s = 0.f, dp = 0.f;
    for (int i = 0; i < hd; ++i) {
      s = fmaf(qs[w][i], to_f(kr[i]), s);
      dp = fmaf(dos[w][i], to_f(vr[i]), dp);
    }
    float p = expf(s * scale - L);
    ds[j] = p * (dp - D);
  }
  __syncwarp();
  for (int i = lane; i < hd; i += 32) {
    float acc = 0.f;
    for (int j = j0; j <= t; ++j) acc = fmaf(ds[j], to_f(k[kvbase + int64_t(j) * hd + i]), acc);
    gs[w][i] = acc * scale;
  }
  __syncwarp();
  if (lane == 0) Dbuf[int64_t(bh) * Tn + t] = D;
  const int half = hd / 2;
  norm_rope_bwd_row<T>(gs[w], qs[w], rq[int64_t(bh) * Tn + t], qk_norm, cos_t + t * half,
                       sin_t + t * half, hd, lane, dqkv + n * Q + h * hd);
}

// dK, dV of one key row j of key/value head (b, hk): the sum over the query
// heads that share it and over the queries t in [j, j + W) that see it.
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
    attn_bwd_dkv_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                      const T* __restrict__ dO, const float* __restrict__ lse,
                      const float* __restrict__ Dbuf, const float* __restrict__ rk,
                      const float* __restrict__ cos_t, const float* __restrict__ sin_t,
                      T* __restrict__ dqkv, int H, int Hkv, int Tn, int hd, int W, float scale,
                      int qk_norm) {
  extern __shared__ float smem[];
  __shared__ float ks[kWarps][kMaxHd], vs[kWarps][kMaxHd], gs[kWarps][kMaxHd];
  constexpr int kPer = kMaxHd / 32;  // head-dim entries per lane
  const int w = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int j = blockIdx.x * kWarps + w;
  const int bkv = blockIdx.y;  // b * Hkv + hk
  if (j >= Tn) return;
  const int b = bkv / Hkv, hk = bkv % Hkv, rep = H / Hkv, d = H * hd, Q = d + 2 * Hkv * hd;
  float* ps = smem + (2 * w) * Tn;
  float* dss = smem + (2 * w + 1) * Tn;
  const int64_t kvbase = int64_t(bkv) * Tn * hd;
  const int i_end = int(min(int64_t(Tn), int64_t(j) + W));  // queries j .. i_end-1 see key j
  for (int i = lane; i < hd; i += 32) {
    ks[w][i] = to_f(k[kvbase + int64_t(j) * hd + i]);
    vs[w][i] = to_f(v[kvbase + int64_t(j) * hd + i]);
  }
  __syncwarp();
  float dv[kPer], dk[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) dv[u] = dk[u] = 0.f;
  for (int g = 0; g < rep; ++g) {
    const int h = hk * rep + g;
    const int64_t bh = int64_t(b) * H + h;
    const int64_t base = bh * Tn * hd;
    for (int i = j + lane; i < i_end; i += 32) {
      const T* qr = q + base + int64_t(i) * hd;
      const T* dr = dO + (int64_t(b) * Tn + i) * d + h * hd;
      float s = 0.f, dp = 0.f;
      for (int e = 0; e < hd; ++e) {
        s = fmaf(to_f(qr[e]), ks[w][e], s);
        dp = fmaf(to_f(dr[e]), vs[w][e], dp);
      }
      float p = expf(s * scale - lse[bh * Tn + i]);
      ps[i] = p;
      dss[i] = p * (dp - Dbuf[bh * Tn + i]);
    }
    __syncwarp();
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = lane + 32 * u;
      if (e >= hd) break;
      for (int i = j; i < i_end; ++i) {
        dv[u] = fmaf(ps[i], to_f(dO[(int64_t(b) * Tn + i) * d + h * hd + e]), dv[u]);
        dk[u] = fmaf(dss[i], to_f(q[base + int64_t(i) * hd + e]), dk[u]);
      }
    }
    __syncwarp();
  }
  const int64_t n = int64_t(b) * Tn + j;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int e = lane + 32 * u;
    if (e >= hd) break;
    dqkv[n * Q + d + Hkv * hd + hk * hd + e] = from_f<T>(dv[u]);
    gs[w][e] = dk[u] * scale;
  }
  __syncwarp();
  const int half = hd / 2;
  norm_rope_bwd_row<T>(gs[w], ks[w], rk[int64_t(bkv) * Tn + j], qk_norm, cos_t + j * half,
                       sin_t + j * half, hd, lane, dqkv + n * Q + d + hk * hd);
}

template <typename T>
static int attn_fwd_t(const gpt_config& c, const void* q, const void* k, const void* v, void* o,
                      float* lse, cudaStream_t st) {
  const int Tn = c.seq_len;
  size_t smem = size_t(kWarps) * Tn * 4;
  auto kern = attn_fwd_simt<T>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
      cudaSuccess)
    return 1;
  dim3 grid(ceil_div(Tn, kWarps), c.batch * c.n_head);
  kern<<<grid, kWarps * 32, smem, st>>>((const T*)q, (const T*)k, (const T*)v, (T*)o, lse,
                                       c.n_head, c.n_kv_head, Tn, c.head_dim, window_span(c),
                                       1.f / sqrtf(float(c.head_dim)));
  return last_launch_rc();
}

template <typename T>
static int attn_bwd_t(const gpt_config& c, const void* q, const void* k, const void* v,
                      const void* o, const void* dO, const float* lse, const float* rq,
                      const float* rk, const float* cos_t, const float* sin_t, float* Dbuf,
                      void* dqkv, cudaStream_t st) {
  const int Tn = c.seq_len;
  const float scale = 1.f / sqrtf(float(c.head_dim));
  dim3 grid(ceil_div(Tn, kWarps), c.batch * c.n_head);
  dim3 grid_kv(ceil_div(Tn, kWarps), c.batch * c.n_kv_head);
  size_t smem1 = size_t(kWarps) * Tn * 4;
  auto k1 = attn_bwd_dq_simt<T>;
  if (cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem1)) !=
      cudaSuccess)
    return 1;
  k1<<<grid, kWarps * 32, smem1, st>>>((const T*)q, (const T*)k, (const T*)v, (const T*)o,
                                      (const T*)dO, lse, rq, cos_t, sin_t, Dbuf, (T*)dqkv,
                                      c.n_head, c.n_kv_head, Tn, c.head_dim, window_span(c), scale,
                                      c.qk_norm);
  size_t smem2 = size_t(2 * kWarps) * Tn * 4;
  auto k2 = attn_bwd_dkv_simt<T>;
  if (cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem2)) !=
      cudaSuccess)
    return 1;
  k2<<<grid_kv, kWarps * 32, smem2, st>>>((const T*)q, (const T*)k, (const T*)v, (const T*)dO,
                                         lse, Dbuf, rk, cos_t, sin_t, (T*)dqkv, c.n_head,
                                         c.n_kv_head, Tn, c.head_dim, window_span(c), scale,
                                         c.qk_norm);
  return last_launch_rc();
}

int launch_attn_fwd_simt(const gpt_config& c, const void* q, const void* k, const void* v,
                         void* o, float* lse, void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  return c.dtype == GPT_BF16 ? attn_fwd_t<__nv_bfloat16>(c, q, k, v, o, lse, st)
                             : attn_fwd_t<float>(c, q, k, v, o, lse, st);
}

int launch_attn_bwd_simt(const gpt_config& c, const void* q, const void* k, const void* v,
                         const void* o, const void* dO, const float* lse, const float* rq,
                         const float* rk, const float* cos_t, const float* sin_t, float* Dbuf,
                         void* dqkv, void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  return c.dtype == GPT_BF16
             ? attn_bwd_t<__nv_bfloat16>(c, q, k, v, o, dO, lse, rq, rk, cos_t, sin_t, Dbuf,
                                         dqkv, st)
             : attn_bwd_t<float>(c, q, k, v, o, dO, lse, rq, rk, cos_t, sin_t, Dbuf, dqkv, st);
}

}  // namespace gpt
