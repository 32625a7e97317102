// Causal flash attention forward on the sm_100a tensor cores.
//
// o = softmax(q k^T / sqrt(hd), keys <= query) v, per (batch, head); q, k, v
// head-major [B*H*T, hd] bf16 (q, k already rotated and normalised), o
// token-major [B*T, H*hd] bf16, lse [B*H*T] fp32 = log sum_j exp(s_ij).
//
// One CTA per (128-query tile, batch*head), the longest causal rows first.
//   warp 0      TMA: the Q tile once, K_j / V_j tiles through a 2-stage ring;
//   warp 1      one thread issues S_j = Q K_j^T (M=128, N=128, K=hd) into one of
//               two TMEM score buffers, and O += P_j V_j (M=128, N=hd,
//               K=128) into the TMEM output accumulator, so S_{j+1} runs during
//               softmax(S_j) and P_j V_j during softmax(S_{j+1});
//   warps 2..5  thread = query row: running max and sum in base 2, P_j as bf16
//               into shared memory in the 128B-swizzled K-major layout the
//               PV MMA reads.  O accumulates in TMEM (O += P_j V_j); a row's O
//               and sum are rescaled (tcgen05.ld/st) only when its max grows
//               by more than 2^8 over the reference max they share, so the
//               result is exact and most tiles need no O round trip.
// All waits are bounded (GPT_ETIMEOUT in the status word).
#include <cudaTypedefs.h>

#include "device_common.cuh"
#include "tc_ptx.cuh"

namespace gpt {

namespace {
constexpr int BQ = 128, BKV = 128;
constexpr int kThreads = 192;
constexpr uint64_t kWaitNs = 2000000000ull;

template <int HD>
struct FwdSmem {
  static constexpr uint32_t TILE = BQ * HD * 2;  // one 128-row bf16 tile (Q, K, V or P)
  static constexpr uint32_t P_BYTES = BQ * BKV * 2;
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t K_OFF = Q_OFF + TILE;          // 2 stages
  static constexpr uint32_t V_OFF = K_OFF + 2 * TILE;      // 2 stages
  static constexpr uint32_t P_OFF = V_OFF + 2 * TILE;
  static constexpr uint32_t BAR_OFF = P_OFF + P_BYTES;
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;  // + barriers + alignment slack
};

struct FwdBars {
  uint64_t q_full;
  uint64_t kv_full[2];
  uint64_t kv_empty[2];
  uint64_t s_full[2];
  uint64_t p_ready;
  uint64_t pv_full;
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
}  // namespace

template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                       const __grid_constant__ CUtensorMap map_k,
                       const __grid_constant__ CUtensorMap map_v, __nv_bfloat16* __restrict__ o,
                       float* __restrict__ lse, int H, int T, float scale_log2,
                       int32_t* status) {
  using S = FwdSmem<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + S::BAR_OFF);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int n_qt = (T + BQ - 1) / BQ;
  const int BH = gridDim.x / n_qt;
  const int qt = n_qt - 1 - int(blockIdx.x) / BH;  // longest rows first
  const int bh = int(blockIdx.x) % BH;
  const int q0 = qt * BQ;
  const int n_kv = qt + 1;                          // causal: KV tiles 0..qt
  const int row_base = bh * T;                      // first row of this (b, h) in q/k/v
  constexpr uint32_t HD_CHUNK = BQ * 128;           // bytes of one 64-column chunk of a tile
  constexpr int NCH = HD / 64;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->kv_full[s], 1);
      tc::mbar_init(&bars->kv_empty[s], 1);
      tc::mbar_init(&bars->s_full[s], 1);
    }
    tc::mbar_init(&bars->p_ready, 128);
    tc::mbar_init(&bars->pv_full, 1);
    tc::mbar_init(&bars->done, 1);
    bars->abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  // TMEM columns: S buffers at 0 and 128, O accumulator at 256
  const uint32_t t_o = tmem + 256;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t issued = 0, last_par = 0;
      tc::mbar_arrive_expect_tx(&bars->q_full, S::TILE);
#pragma unroll
      for (int c = 0; c < NCH; ++c)
        tc::tma_load_2d(smem + S::Q_OFF + c * HD_CHUNK, &map_q, &bars->q_full, c * 64,
                        row_base + q0);
      for (int j = 0; j < n_kv; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!tc::mbar_wait_bounded(&bars->kv_empty[st], ph ^ 1, abort, kWaitNs)) {
          record_status(status, GPT_ETIMEOUT, K_ATTN, 10);
          *abort = 1;
          break;
        }
        tc::mbar_arrive_expect_tx(&bars->kv_full[st], 2 * S::TILE);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          tc::tma_load_2d(smem + S::K_OFF + st * S::TILE + c * HD_CHUNK, &map_k, &bars->kv_full[st],
                          c * 64, row_base + j * BKV);
          tc::tma_load_2d(smem + S::V_OFF + st * S::TILE + c * HD_CHUNK, &map_v, &bars->kv_full[st],
                          c * 64, row_base + j * BKV);
        }
        issued |= 1u << st;
        last_par = (last_par & ~(1u << st)) | (ph << st);
      }
      if (*abort) {
        tc::mbar_wait_bounded(&bars->q_full, 0, nullptr, kWaitNs);
        for (int s = 0; s < 2; ++s)
          if (issued >> s & 1) tc::mbar_wait_bounded(&bars->kv_full[s], (last_par >> s) & 1, nullptr, kWaitNs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(BQ, BKV, false, false);
      constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(BQ, HD, false, true);
      const uint32_t q_addr = tc::smem_u32(smem + S::Q_OFF);
      const uint32_t p_addr = tc::smem_u32(smem + S::P_OFF);
      bool ok = tc::mbar_wait_bounded(&bars->q_full, 0, abort, kWaitNs);
      bool issued_any = false;
      auto issue_pv = [&](int j) -> bool {
        if (!tc::mbar_wait_bounded(&bars->p_ready, j & 1, abort, kWaitNs)) return false;
        tc::tc_fence_after();
        const uint32_t v_addr = tc::smem_u32(smem + S::V_OFF + (j & 1) * S::TILE);
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k) {
          const uint64_t da = tc::smem_desc_sw128(p_addr + (k >> 2) * (BQ * 128) + (k & 3) * 32, 16);
          const uint64_t db = tc::smem_desc_sw128(v_addr + k * 2048, HD_CHUNK);
          tc::mma_bf16_ss(t_o, da, db, idesc_pv, (j | k) != 0);
        }
        tc::mma_commit(&bars->pv_full);
        tc::mma_commit(&bars->kv_empty[j & 1]);
        return true;
      };
      for (int j = 0; ok && j < n_kv; ++j) {
        const int st = j & 1;
        if (!tc::mbar_wait_bounded(&bars->kv_full[st], (j >> 1) & 1, abort, kWaitNs)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t k_addr = tc::smem_u32(smem + S::K_OFF + st * S::TILE);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t off = (k >> 2) * HD_CHUNK + (k & 3) * 32;
          tc::mma_bf16_ss(tmem + st * 128, tc::smem_desc_sw128(q_addr + off, 16),
                          tc::smem_desc_sw128(k_addr + off, 16), idesc_s, k != 0);
        }
        issued_any = true;
        tc::mma_commit(&bars->s_full[st]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && n_kv >= 1) ok = issue_pv(n_kv - 1);
      if (!ok) {
        record_status(status, GPT_ETIMEOUT, K_ATTN, 11);
        *abort = 1;
      }
      if (issued_any) {
        tc::mma_commit(&bars->done);
        tc::mbar_wait_bounded(&bars->done, 0, nullptr, kWaitNs);
      }
    }
  } else {
    // softmax warps: thread = query row
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int q = q0 + r;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    uint8_t* p_tile = smem + S::P_OFF;
    float m_ref = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {
      const int st = j & 1;
      const uint32_t t_s = tmem + st * 128 + lane_off;
      ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->s_full[st], (j >> 1) & 1, abort, kWaitNs));
      if (!ok) break;
      tc::tc_fence_after();
      const bool diag = j == qt;
      const int k0 = j * BKV;
      // pass 1: row max of the scaled, masked scores (base-2 units)
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < BKV / 32; ++c) {
        uint32_t u[32];
        tc::tmem_ld_32x32b_x32(t_s + c * 32, u);
        tc::tmem_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int key = k0 + c * 32 + jj;
          float sv = __uint_as_float(u[jj]) * scale_log2;
          if ((diag && key > q) || key >= T) sv = -INFINITY;
          mx = fmaxf(mx, sv);
        }
      }
      // P_{j-1} V_{j-1} must have finished before P_j overwrites the P tile
      if (j > 0) {
        ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->pv_full, (j - 1) & 1, abort, kWaitNs));
        if (!ok) break;
        tc::tc_fence_after();
      }
      // move the reference max only when it grows by more than 2^8 (or on the first tile)
      const bool grow = mx > m_ref + 8.f;
      const float factor = grow ? ex2(m_ref - mx) : 1.f;  // 0 on the first tile
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll
        for (int c = 0; c < HD / 16; ++c) {
          uint32_t u[16];
          tc::tmem_ld_32x32b_x16(t_o + lane_off + c * 16, u);
          tc::tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) u[jj] = __float_as_uint(__uint_as_float(u[jj]) * factor);
          tc::tmem_st_32x32b_x16(t_o + lane_off + c * 16, u);
        }
        tc::tmem_wait_st();
      }
      if (grow) {
        l_run *= factor;
        m_ref = mx;
      }
      // pass 2: P = 2^(s - m_ref) as bf16 into the swizzled P tile; running sum
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < BKV / 16; ++c) {
        uint32_t u[16];
        tc::tmem_ld_32x32b_x16(t_s + c * 16, u);
        tc::tmem_wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int jj = 0; jj < 16; jj += 2) {
          const int key = k0 + c * 16 + jj;
          float s0 = __uint_as_float(u[jj]) * scale_log2;
          float s1 = __uint_as_float(u[jj + 1]) * scale_log2;
          if ((diag && key > q) || key >= T) s0 = -INFINITY;
          if ((diag && key + 1 > q) || key + 1 >= T) s1 = -INFINITY;
          const float p0 = ex2(s0 - m_ref), p1 = ex2(s1 - m_ref);
          lsum += p0 + p1;
          pk[jj / 2] = pack2(p0, p1);
        }
        // keys c*16 .. c*16+15: chunk c/4 of 64 keys, 16-byte units (c%4)*2 and +1
        uint8_t* rowp = p_tile + (c >> 2) * (BQ * 128) + r * 128;
#pragma unroll
        for (int v2 = 0; v2 < 2; ++v2) {
          const int unit = (c & 3) * 2 + v2;
          uint4 val = make_uint4(pk[v2 * 4], pk[v2 * 4 + 1], pk[v2 * 4 + 2], pk[v2 * 4 + 3]);
          *reinterpret_cast<uint4*>(rowp + ((unit ^ (r & 7)) << 4)) = val;
        }
      }
      l_run += lsum;
      fence_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(&bars->p_ready);
    }
    if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->pv_full, (n_kv - 1) & 1, abort, kWaitNs));
    if (!ok) {
      if (lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 12);
      *abort = 1;
    } else {
      tc::tc_fence_after();
      const int b = bh / H, h = bh % H;
      const float inv = 1.f / l_run;
      __nv_bfloat16* dst = o + (int64_t(b) * T + q) * (int64_t(H) * HD) + h * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t u[32];
        tc::tmem_ld_32x32b_x32(t_o + lane_off + c * 32, u);
        tc::tmem_wait_ld();
        if (q < T) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 val = make_uint4(
                pack2(__uint_as_float(u[i]) * inv, __uint_as_float(u[i + 1]) * inv),
                pack2(__uint_as_float(u[i + 2]) * inv, __uint_as_float(u[i + 3]) * inv),
                pack2(__uint_as_float(u[i + 4]) * inv, __uint_as_float(u[i + 5]) * inv),
                pack2(__uint_as_float(u[i + 6]) * inv, __uint_as_float(u[i + 7]) * inv));
            *reinterpret_cast<uint4*>(dst + c * 32 + i) = val;
          }
        }
      }
      if (q < T) lse[int64_t(bh) * T + q] = (m_ref + __log2f(l_run)) * 0.69314718055994531f;
    }
  }

  __syncwarp();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [rows, hd] bf16 head-major tensor, box 64 columns x 128 rows, 128B swizzle
bool rows_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t hd) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {hd, rows};
  cuuint64_t strides[1] = {hd * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HD>
int attn_fwd_tc_t(const gpt_config& c, const void* q, const void* k, const void* v, void* o,
                  float* lse, int32_t* status, cudaStream_t st) {
  const uint64_t rows = uint64_t(c.batch) * c.n_head * c.seq_len;
  CUtensorMap mq, mk, mv;
  if (!rows_map(&mq, q, rows, HD) || !rows_map(&mk, k, rows, HD) || !rows_map(&mv, v, rows, HD))
    return 1;
  auto kern = attn_fwd_tc_kernel<HD>;
  const int smem = int(FwdSmem<HD>::BYTES);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 1;
  const int n_qt = (c.seq_len + BQ - 1) / BQ;
  const float scale_log2 = 1.4426950408889634f / sqrtf(float(c.head_dim));
  kern<<<n_qt * c.batch * c.n_head, kThreads, smem, st>>>(
      mq, mk, mv, static_cast<__nv_bfloat16*>(o), lse, c.n_head, c.seq_len, scale_log2, status);
  return last_launch_rc();
}
}  // namespace

int launch_attn_fwd_tc(const gpt_config& c, const void* q, const void* k, const void* v, void* o,
                       float* lse, int32_t* status, void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  return c.head_dim == 128 ? attn_fwd_tc_t<128>(c, q, k, v, o, lse, status, st)
                           : attn_fwd_tc_t<64>(c, q, k, v, o, lse, status, st);
}

// ===========================================================================
// Backward.  With P_ij = exp(s_ij / sqrt(hd) - lse_i) and D_i = dO_i . o_i:
//   dS_ij = P_ij (dO_i . v_j - D_i)
//   dQ_i  = sum_j dS_ij k_j / sqrt(hd)      (kernel attn_dq_tc: CTA = 128 queries)
//   dK_j  = sum_i dS_ij q_i / sqrt(hd)      (kernel attn_dkv_tc: CTA = 128 keys)
//   dV_j  = sum_i P_ij dO_i
// Each kernel owns its outputs, so no sum needs atomics (deterministic).  The
// gradients of q and k then go back through the per-head RMSNorm,
// dx = r (g - y mean(g y)), and the transposed RoPE rotation, and land in the
// [q | k | v] gradient rows [B*T, 3*H*hd].
// ===========================================================================
namespace {

constexpr int kInner = 64;  // inner-loop tile (keys in attn_dq_tc, queries in attn_dkv_tc)

// D_i = dO_i . o_i, one warp per (token, head)
__global__ void attn_rowdot_kernel(const __nv_bfloat16* __restrict__ dO,
                                   const __nv_bfloat16* __restrict__ o, float* __restrict__ D,
                                   int64_t N, int H, int T, int hd) {
  const int64_t w = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (w >= N * H) return;
  const int64_t n = w / H;
  const int h = int(w % H);
  const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(dO + n * H * hd + h * hd);
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(o + n * H * hd + h * hd);
  float s = 0.f;
  for (int i = lane; i < hd / 2; i += 32) {
    float2 x = __bfloat1622float2(a[i]), y = __bfloat1622float2(b[i]);
    s += x.x * y.x + x.y * y.y;
  }
  s = warp_sum(s);
  if (lane == 0) {
    const int64_t bb = n / T, t = n % T;
    D[(bb * H + h) * T + t] = s;
  }
}

struct BwdBars {
  uint64_t fixed_full;     // tiles loaded once per CTA
  uint64_t ring_full[2];
  uint64_t ring_empty[2];
  uint64_t s_full[2];
  uint64_t ds_ready[2];
  uint64_t acc_full;
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

// Gradient w.r.t. one row of q or k, held in TMEM (fp32, HD columns, this
// thread's lane), times `scale`, back through RMSNorm (y: the normalised row
// in global memory, r its 1/rms) and RoPE; written as bf16 to out[0..HD).
template <int HD>
__device__ __forceinline__ void norm_rope_bwd_from_tmem(uint32_t taddr, float scale,
                                                         const __nv_bfloat16* __restrict__ y,
                                                         float r, int qk_norm,
                                                         const float* __restrict__ cosr,
                                                         const float* __restrict__ sinr,
                                                         __nv_bfloat16* __restrict__ out,
                                                         bool write) {
  constexpr int HALF = HD / 2;
  float mean_gy = 0.f;
  if (qk_norm) {
#pragma unroll
    for (int c = 0; c < HD / 16; ++c) {
      uint32_t u[16];
      tc::tmem_ld_32x32b_x16(taddr + c * 16, u);
      tc::tmem_wait_ld();
      if (write) {
        const uint4* yp = reinterpret_cast<const uint4*>(y + c * 16);
        uint4 y0 = yp[0], y1 = yp[1];
        const uint32_t yw[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162*>(&yw[e]);
          float2 yf = __bfloat1622float2(h2);
          mean_gy += __uint_as_float(u[2 * e]) * yf.x + __uint_as_float(u[2 * e + 1]) * yf.y;
        }
      }
    }
    mean_gy *= scale / float(HD);
  }
#pragma unroll
  for (int c = 0; c < HALF / 16; ++c) {
    uint32_t ua[16], ub[16];
    tc::tmem_ld_32x32b_x16(taddr + c * 16, ua);
    tc::tmem_ld_32x32b_x16(taddr + HALF + c * 16, ub);
    tc::tmem_wait_ld();
    if (!write) continue;
    uint32_t pa[8], pb[8];
    const uint4* ya = reinterpret_cast<const uint4*>(y + c * 16);
    const uint4* yb = reinterpret_cast<const uint4*>(y + HALF + c * 16);
    uint4 ya0 = ya[0], ya1 = ya[1], yb0 = yb[0], yb1 = yb[1];
    const uint32_t yaw[8] = {ya0.x, ya0.y, ya0.z, ya0.w, ya1.x, ya1.y, ya1.z, ya1.w};
    const uint32_t ybw[8] = {yb0.x, yb0.y, yb0.z, yb0.w, yb1.x, yb1.y, yb1.z, yb1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float2 yfa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&yaw[e]));
      float2 yfb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ybw[e]));
      float ga0 = __uint_as_float(ua[2 * e]) * scale, ga1 = __uint_as_float(ua[2 * e + 1]) * scale;
      float gb0 = __uint_as_float(ub[2 * e]) * scale, gb1 = __uint_as_float(ub[2 * e + 1]) * scale;
      if (qk_norm) {
        ga0 = r * (ga0 - yfa.x * mean_gy); ga1 = r * (ga1 - yfa.y * mean_gy);
        gb0 = r * (gb0 - yfb.x * mean_gy); gb1 = r * (gb1 - yfb.y * mean_gy);
      }
      const int i0 = c * 16 + 2 * e;
      const float c0 = cosr[i0], s0 = sinr[i0], c1 = cosr[i0 + 1], s1 = sinr[i0 + 1];
      pa[e] = pack2(ga0 * c0 + gb0 * s0, ga1 * c1 + gb1 * s1);
      pb[e] = pack2(-ga0 * s0 + gb0 * c0, -ga1 * s1 + gb1 * c1);
    }
    uint4* oa = reinterpret_cast<uint4*>(out + c * 16);
    uint4* ob = reinterpret_cast<uint4*>(out + HALF + c * 16);
    oa[0] = make_uint4(pa[0], pa[1], pa[2], pa[3]);
    oa[1] = make_uint4(pa[4], pa[5], pa[6], pa[7]);
    ob[0] = make_uint4(pb[0], pb[1], pb[2], pb[3]);
    ob[1] = make_uint4(pb[4], pb[5], pb[6], pb[7]);
  }
}

template <int HD>
struct DqSmem {
  static constexpr uint32_t BIG = 128 * HD * 2;    // 128-row tile
  static constexpr uint32_t SMALL = kInner * HD * 2;
  static constexpr uint32_t DS = 128 * kInner * 2;
  static constexpr uint32_t Q_OFF = 0, DO_OFF = BIG, K_OFF = 2 * BIG;
  static constexpr uint32_t V_OFF = K_OFF + 2 * SMALL;
  static constexpr uint32_t DS_OFF = V_OFF + 2 * SMALL;
  static constexpr uint32_t BAR_OFF = DS_OFF + 2 * DS;
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;
};

}  // namespace

// dQ for 128 queries of one (batch, head), looping over 64-key tiles.
template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_dq_tc_kernel(const __grid_constant__ CUtensorMap map_q128,
                      const __grid_constant__ CUtensorMap map_do128,
                      const __grid_constant__ CUtensorMap map_k64,
                      const __grid_constant__ CUtensorMap map_v64,
                      const __nv_bfloat16* __restrict__ qn, const float* __restrict__ lse,
                      const float* __restrict__ D, const float* __restrict__ rq,
                      const float* __restrict__ cos_t, const float* __restrict__ sin_t,
                      __nv_bfloat16* __restrict__ dqkv, int H, int T, float scale,
                      float scale_log2, int qk_norm, int32_t* status) {
  using S = DqSmem<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + S::BAR_OFF);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int n_qt = (T + 127) / 128;
  const int BH = gridDim.x / n_qt;
  const int qt = n_qt - 1 - int(blockIdx.x) / BH;
  const int bh = int(blockIdx.x) % BH;
  const int b = bh / H, h = bh % H;
  const int q0 = qt * 128;
  const int n_steps = (min(q0 + 128, T) + kInner - 1) / kInner;
  constexpr int NCH = HD / 64;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->fixed_full, 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->ring_full[s], 1);
      tc::mbar_init(&bars->ring_empty[s], 1);
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->ds_ready[s], 128);
    }
    tc::mbar_init(&bars->acc_full, 1);
    tc::mbar_init(&bars->done, 1);
    bars->abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  const uint32_t t_dq = tmem + 256;  // S/dP pairs at 0 and 128 (64 + 64 columns each)

  if (warp == 0) {
    if (lane == 0) {
      uint32_t issued = 0, last_par = 0;
      tc::mbar_arrive_expect_tx(&bars->fixed_full, 2 * S::BIG);
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        tc::tma_load_2d(smem + S::Q_OFF + c * (128 * 128), &map_q128, &bars->fixed_full, c * 64,
                        bh * T + q0);
        tc::tma_load_2d(smem + S::DO_OFF + c * (128 * 128), &map_do128, &bars->fixed_full,
                        h * HD + c * 64, b * T + q0);
      }
      for (int j = 0; j < n_steps; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!tc::mbar_wait_bounded(&bars->ring_empty[st], ph ^ 1, abort, kWaitNs)) {
          record_status(status, GPT_ETIMEOUT, K_ATTN, 20);
          *abort = 1;
          break;
        }
        tc::mbar_arrive_expect_tx(&bars->ring_full[st], 2 * S::SMALL);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          tc::tma_load_2d(smem + S::K_OFF + st * S::SMALL + c * (kInner * 128), &map_k64,
                          &bars->ring_full[st], c * 64, bh * T + j * kInner);
          tc::tma_load_2d(smem + S::V_OFF + st * S::SMALL + c * (kInner * 128), &map_v64,
                          &bars->ring_full[st], c * 64, bh * T + j * kInner);
        }
        issued |= 1u << st;
        last_par = (last_par & ~(1u << st)) | (ph << st);
      }
      if (*abort) {
        tc::mbar_wait_bounded(&bars->fixed_full, 0, nullptr, kWaitNs);
        for (int s = 0; s < 2; ++s)
          if (issued >> s & 1) tc::mbar_wait_bounded(&bars->ring_full[s], (last_par >> s) & 1, nullptr, kWaitNs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, kInner, false, false);
      constexpr uint32_t idesc_dq = tc::idesc_bf16_f32(128, HD, false, true);
      const uint32_t q_addr = tc::smem_u32(smem + S::Q_OFF);
      const uint32_t do_addr = tc::smem_u32(smem + S::DO_OFF);
      bool ok = tc::mbar_wait_bounded(&bars->fixed_full, 0, abort, kWaitNs);
      bool issued_any = false;
      auto issue_dq = [&](int j) -> bool {
        if (!tc::mbar_wait_bounded(&bars->ds_ready[j & 1], (j >> 1) & 1, abort, kWaitNs)) return false;
        tc::tc_fence_after();
        const uint32_t ds_addr = tc::smem_u32(smem + S::DS_OFF + (j & 1) * S::DS);
        const uint32_t k_addr = tc::smem_u32(smem + S::K_OFF + (j & 1) * S::SMALL);
#pragma unroll
        for (int k = 0; k < kInner / 16; ++k)
          tc::mma_bf16_ss(t_dq, tc::smem_desc_sw128(ds_addr + k * 32, 16),
                          tc::smem_desc_sw128(k_addr + k * 2048, kInner * 128), idesc_dq,
                          (j | k) != 0);
        tc::mma_commit(&bars->ring_empty[j & 1]);
        return true;
      };
      for (int j = 0; ok && j < n_steps; ++j) {
        const int st = j & 1;
        if (!tc::mbar_wait_bounded(&bars->ring_full[st], (j >> 1) & 1, abort, kWaitNs)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t k_addr = tc::smem_u32(smem + S::K_OFF + st * S::SMALL);
        const uint32_t v_addr = tc::smem_u32(smem + S::V_OFF + st * S::SMALL);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t big = (k >> 2) * (128 * 128) + (k & 3) * 32;
          const uint32_t small = (k >> 2) * (kInner * 128) + (k & 3) * 32;
          tc::mma_bf16_ss(tmem + st * 128, tc::smem_desc_sw128(q_addr + big, 16),
                          tc::smem_desc_sw128(k_addr + small, 16), idesc_s, k != 0);
          tc::mma_bf16_ss(tmem + st * 128 + kInner, tc::smem_desc_sw128(do_addr + big, 16),
                          tc::smem_desc_sw128(v_addr + small, 16), idesc_s, k != 0);
        }
        issued_any = true;
        tc::mma_commit(&bars->s_full[st]);
        if (j >= 1 && !issue_dq(j - 1)) { ok = false; break; }
      }
      if (ok && n_steps >= 1) ok = issue_dq(n_steps - 1);
      if (ok) tc::mma_commit(&bars->acc_full);
      if (!ok) {
        record_status(status, GPT_ETIMEOUT, K_ATTN, 21);
        *abort = 1;
      }
      if (issued_any) {
        tc::mma_commit(&bars->done);
        tc::mbar_wait_bounded(&bars->done, 0, nullptr, kWaitNs);
      }
    }
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int q = q0 + r;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const bool qv = q < T;
    const float lse2 = qv ? lse[int64_t(bh) * T + q] * 1.4426950408889634f : 0.f;
    const float Dq = qv ? D[int64_t(bh) * T + q] : 0.f;
    bool ok = true;
    for (int j = 0; j < n_steps && ok; ++j) {
      const int st = j & 1;
      ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->s_full[st], (j >> 1) & 1, abort, kWaitNs));
      if (!ok) break;
      tc::tc_fence_after();
      const int k0 = j * kInner;
      uint8_t* rowp = smem + S::DS_OFF + st * S::DS + r * 128;
#pragma unroll
      for (int c = 0; c < kInner / 16; ++c) {
        uint32_t us[16], up[16];
        tc::tmem_ld_32x32b_x16(tmem + st * 128 + lane_off + c * 16, us);
        tc::tmem_ld_32x32b_x16(tmem + st * 128 + kInner + lane_off + c * 16, up);
        tc::tmem_wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const int key = k0 + c * 16 + e;
          float p0 = ex2(__uint_as_float(us[e]) * scale_log2 - lse2);
          float p1 = ex2(__uint_as_float(us[e + 1]) * scale_log2 - lse2);
          if (key > q || key >= T || !qv) p0 = 0.f;
          if (key + 1 > q || key + 1 >= T || !qv) p1 = 0.f;
          pk[e / 2] = pack2(p0 * (__uint_as_float(up[e]) - Dq), p1 * (__uint_as_float(up[e + 1]) - Dq));
        }
#pragma unroll
        for (int v2 = 0; v2 < 2; ++v2) {
          const int unit = c * 2 + v2;
          *reinterpret_cast<uint4*>(rowp + ((unit ^ (r & 7)) << 4)) =
              make_uint4(pk[v2 * 4], pk[v2 * 4 + 1], pk[v2 * 4 + 2], pk[v2 * 4 + 3]);
        }
      }
      fence_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(&bars->ds_ready[st]);
    }
    if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->acc_full, 0, abort, kWaitNs));
    if (!ok) {
      if (lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 22);
      *abort = 1;
    } else {
      tc::tc_fence_after();
      const int d = H * HD;
      const int tq = qv ? q : 0;
      norm_rope_bwd_from_tmem<HD>(t_dq + lane_off, scale, qn + (int64_t(bh) * T + tq) * HD,
                                  qv ? rq[int64_t(bh) * T + q] : 0.f, qk_norm,
                                  cos_t + tq * (HD / 2), sin_t + tq * (HD / 2),
                                  dqkv + (int64_t(b) * T + tq) * 3 * d + h * HD, qv);
    }
  }

  __syncwarp();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

namespace {
template <int HD>
struct DkvSmem {
  static constexpr uint32_t BIG = 128 * HD * 2;
  static constexpr uint32_t SMALL = kInner * HD * 2;
  static constexpr uint32_t PT = 128 * kInner * 2;
  static constexpr uint32_t K_OFF = 0, V_OFF = BIG, Q_OFF = 2 * BIG;
  static constexpr uint32_t DO_OFF = Q_OFF + 2 * SMALL;
  static constexpr uint32_t P_OFF = DO_OFF + 2 * SMALL;
  static constexpr uint32_t DS_OFF = P_OFF + 2 * PT;
  static constexpr uint32_t BAR_OFF = DS_OFF + 2 * PT;
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;
};
}  // namespace

// dK, dV for 128 keys of one (batch, head), looping over 64-query tiles.
template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_dkv_tc_kernel(const __grid_constant__ CUtensorMap map_k128,
                       const __grid_constant__ CUtensorMap map_v128,
                       const __grid_constant__ CUtensorMap map_q64,
                       const __grid_constant__ CUtensorMap map_do64,
                       const __nv_bfloat16* __restrict__ kn, const float* __restrict__ lse,
                       const float* __restrict__ D, const float* __restrict__ rk,
                       const float* __restrict__ cos_t, const float* __restrict__ sin_t,
                       __nv_bfloat16* __restrict__ dqkv, int H, int T, float scale,
                       float scale_log2, int qk_norm, int32_t* status) {
  using S = DkvSmem<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + S::BAR_OFF);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int n_kt = (T + 127) / 128;
  const int BH = gridDim.x / n_kt;
  const int kt = int(blockIdx.x) / BH;  // key tile 0 has the most queries: first
  const int bh = int(blockIdx.x) % BH;
  const int b = bh / H, h = bh % H;
  const int k0 = kt * 128;
  const int i_begin = k0 / kInner;
  const int n_steps = (T + kInner - 1) / kInner - i_begin;
  constexpr int NCH = HD / 64;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->fixed_full, 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->ring_full[s], 1);
      tc::mbar_init(&bars->ring_empty[s], 1);
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->ds_ready[s], 128);
    }
    tc::mbar_init(&bars->acc_full, 1);
    tc::mbar_init(&bars->done, 1);
    bars->abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  const uint32_t t_dv = tmem + 256, t_dk = tmem + 256 + HD;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t issued = 0, last_par = 0;
      tc::mbar_arrive_expect_tx(&bars->fixed_full, 2 * S::BIG);
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        tc::tma_load_2d(smem + S::K_OFF + c * (128 * 128), &map_k128, &bars->fixed_full, c * 64,
                        bh * T + k0);
        tc::tma_load_2d(smem + S::V_OFF + c * (128 * 128), &map_v128, &bars->fixed_full, c * 64,
                        bh * T + k0);
      }
      for (int j = 0; j < n_steps; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int qs = (i_begin + j) * kInner;
        if (!tc::mbar_wait_bounded(&bars->ring_empty[st], ph ^ 1, abort, kWaitNs)) {
          record_status(status, GPT_ETIMEOUT, K_ATTN, 30);
          *abort = 1;
          break;
        }
        tc::mbar_arrive_expect_tx(&bars->ring_full[st], 2 * S::SMALL);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          tc::tma_load_2d(smem + S::Q_OFF + st * S::SMALL + c * (kInner * 128), &map_q64,
                          &bars->ring_full[st], c * 64, bh * T + qs);
          tc::tma_load_2d(smem + S::DO_OFF + st * S::SMALL + c * (kInner * 128), &map_do64,
                          &bars->ring_full[st], h * HD + c * 64, b * T + qs);
        }
        issued |= 1u << st;
        last_par = (last_par & ~(1u << st)) | (ph << st);
      }
      if (*abort) {
        tc::mbar_wait_bounded(&bars->fixed_full, 0, nullptr, kWaitNs);
        for (int s = 0; s < 2; ++s)
          if (issued >> s & 1) tc::mbar_wait_bounded(&bars->ring_full[s], (last_par >> s) & 1, nullptr, kWaitNs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, kInner, false, false);
      constexpr uint32_t idesc_acc = tc::idesc_bf16_f32(128, HD, false, true);
      const uint32_t k_addr = tc::smem_u32(smem + S::K_OFF);
      const uint32_t v_addr = tc::smem_u32(smem + S::V_OFF);
      bool ok = tc::mbar_wait_bounded(&bars->fixed_full, 0, abort, kWaitNs);
      bool issued_any = false;
      auto issue_acc = [&](int j) -> bool {
        if (!tc::mbar_wait_bounded(&bars->ds_ready[j & 1], (j >> 1) & 1, abort, kWaitNs)) return false;
        tc::tc_fence_after();
        const uint32_t p_addr = tc::smem_u32(smem + S::P_OFF + (j & 1) * S::PT);
        const uint32_t ds_addr = tc::smem_u32(smem + S::DS_OFF + (j & 1) * S::PT);
        const uint32_t q_addr = tc::smem_u32(smem + S::Q_OFF + (j & 1) * S::SMALL);
        const uint32_t do_addr = tc::smem_u32(smem + S::DO_OFF + (j & 1) * S::SMALL);
#pragma unroll
        for (int k = 0; k < kInner / 16; ++k) {
          tc::mma_bf16_ss(t_dv, tc::smem_desc_sw128(p_addr + k * 32, 16),
                          tc::smem_desc_sw128(do_addr + k * 2048, kInner * 128), idesc_acc,
                          (j | k) != 0);
          tc::mma_bf16_ss(t_dk, tc::smem_desc_sw128(ds_addr + k * 32, 16),
                          tc::smem_desc_sw128(q_addr + k * 2048, kInner * 128), idesc_acc,
                          (j | k) != 0);
        }
        tc::mma_commit(&bars->ring_empty[j & 1]);
        return true;
      };
      for (int j = 0; ok && j < n_steps; ++j) {
        const int st = j & 1;
        if (!tc::mbar_wait_bounded(&bars->ring_full[st], (j >> 1) & 1, abort, kWaitNs)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t q_addr = tc::smem_u32(smem + S::Q_OFF + st * S::SMALL);
        const uint32_t do_addr = tc::smem_u32(smem + S::DO_OFF + st * S::SMALL);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t big = (k >> 2) * (128 * 128) + (k & 3) * 32;
          const uint32_t small = (k >> 2) * (kInner * 128) + (k & 3) * 32;
          tc::mma_bf16_ss(tmem + st * 128, tc::smem_desc_sw128(k_addr + big, 16),
                          tc::smem_desc_sw128(q_addr + small, 16), idesc_s, k != 0);
          tc::mma_bf16_ss(tmem + st * 128 + kInner, tc::smem_desc_sw128(v_addr + big, 16),
                          tc::smem_desc_sw128(do_addr + small, 16), idesc_s, k != 0);
        }
        issued_any = true;
        tc::mma_commit(&bars->s_full[st]);
        if (j >= 1 && !issue_acc(j - 1)) { ok = false; break; }
      }
      if (ok && n_steps >= 1) ok = issue_acc(n_steps - 1);
      if (ok) tc::mma_commit(&bars->acc_full);
      if (!ok) {
        record_status(status, GPT_ETIMEOUT, K_ATTN, 31);
        *abort = 1;
      }
      if (issued_any) {
        tc::mma_commit(&bars->done);
        tc::mbar_wait_bounded(&bars->done, 0, nullptr, kWaitNs);
      }
    }
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int key = k0 + r;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    bool ok = true;
    for (int j = 0; j < n_steps && ok; ++j) {
      const int st = j & 1;
      const int qs = (i_begin + j) * kInner;
      ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->s_full[st], (j >> 1) & 1, abort, kWaitNs));
      if (!ok) break;
      tc::tc_fence_after();
      uint8_t* prow = smem + S::P_OFF + st * S::PT + r * 128;
      uint8_t* drow = smem + S::DS_OFF + st * S::PT + r * 128;
#pragma unroll
      for (int c = 0; c < kInner / 16; ++c) {
        uint32_t us[16], up[16];
        tc::tmem_ld_32x32b_x16(tmem + st * 128 + lane_off + c * 16, us);
        tc::tmem_ld_32x32b_x16(tmem + st * 128 + kInner + lane_off + c * 16, up);
        tc::tmem_wait_ld();
        uint32_t pp[8], pd[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          // lse (base 2) and D of queries qa, qa+1: the same address across the warp
          const int qa = qs + c * 16 + e;
          const int64_t ia = int64_t(bh) * T + min(qa, T - 1);
          const int64_t ib = int64_t(bh) * T + min(qa + 1, T - 1);
          float p0 = ex2(__uint_as_float(us[e]) * scale_log2 - __ldg(lse + ia) * 1.4426950408889634f);
          float p1 = ex2(__uint_as_float(us[e + 1]) * scale_log2 - __ldg(lse + ib) * 1.4426950408889634f);
          if (qa < key || qa >= T || key >= T) p0 = 0.f;
          if (qa + 1 < key || qa + 1 >= T || key >= T) p1 = 0.f;
          pp[e / 2] = pack2(p0, p1);
          pd[e / 2] = pack2(p0 * (__uint_as_float(up[e]) - __ldg(D + ia)),
                            p1 * (__uint_as_float(up[e + 1]) - __ldg(D + ib)));
        }
#pragma unroll
        for (int v2 = 0; v2 < 2; ++v2) {
          const int off = ((c * 2 + v2) ^ (r & 7)) << 4;
          *reinterpret_cast<uint4*>(prow + off) = make_uint4(pp[v2 * 4], pp[v2 * 4 + 1], pp[v2 * 4 + 2], pp[v2 * 4 + 3]);
          *reinterpret_cast<uint4*>(drow + off) = make_uint4(pd[v2 * 4], pd[v2 * 4 + 1], pd[v2 * 4 + 2], pd[v2 * 4 + 3]);
        }
      }
      fence_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(&bars->ds_ready[st]);
    }
    if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->acc_full, 0, abort, kWaitNs));
    if (!ok) {
      if (lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 32);
      *abort = 1;
    } else {
      tc::tc_fence_after();
      const int d = H * HD;
      const bool kv = key < T;
      const int tk = kv ? key : 0;
      __nv_bfloat16* row = dqkv + (int64_t(b) * T + tk) * 3 * d;
      // dV
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t u[32];
        tc::tmem_ld_32x32b_x32(t_dv + lane_off + c * 32, u);
        tc::tmem_wait_ld();
        if (kv) {
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            *reinterpret_cast<uint4*>(row + 2 * d + h * HD + c * 32 + i) = make_uint4(
                pack2(__uint_as_float(u[i]), __uint_as_float(u[i + 1])),
                pack2(__uint_as_float(u[i + 2]), __uint_as_float(u[i + 3])),
                pack2(__uint_as_float(u[i + 4]), __uint_as_float(u[i + 5])),
                pack2(__uint_as_float(u[i + 6]), __uint_as_float(u[i + 7])));
        }
      }
      norm_rope_bwd_from_tmem<HD>(t_dk + lane_off, scale, kn + (int64_t(bh) * T + tk) * HD,
                                  kv ? rk[int64_t(bh) * T + key] : 0.f, qk_norm,
                                  cos_t + tk * (HD / 2), sin_t + tk * (HD / 2), row + d + h * HD,
                                  kv);
    }
  }

  __syncwarp();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
namespace {
// [rows, cols] bf16 row-major tensor (row pitch `ld` elements), box 64 x box_rows
bool tile_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
              uint32_t box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HD>
int attn_bwd_tc_t(const gpt_config& c, const void* q, const void* k, const void* v, const void* o,
                  const void* dO, const float* lse, const float* rq, const float* rk,
                  const float* cos_t, const float* sin_t, float* Dbuf, void* dqkv,
                  int32_t* status, cudaStream_t st) {
  const int H = c.n_head, T = c.seq_len, B = c.batch, d = H * HD;
  const uint64_t rows = uint64_t(B) * H * T, ntok = uint64_t(B) * T;
  const int64_t N = int64_t(B) * T;
  attn_rowdot_kernel<<<ceil_div(N * H, 8), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(dO), static_cast<const __nv_bfloat16*>(o), Dbuf, N, H, T, HD);
  CUtensorMap q128, do128, k64, v64, k128, v128, q64, do64;
  bool ok = tile_map(&q128, q, rows, HD, HD, 128) && tile_map(&do128, dO, ntok, d, d, 128) &&
            tile_map(&k64, k, rows, HD, HD, 64) && tile_map(&v64, v, rows, HD, HD, 64) &&
            tile_map(&k128, k, rows, HD, HD, 128) && tile_map(&v128, v, rows, HD, HD, 128) &&
            tile_map(&q64, q, rows, HD, HD, 64) && tile_map(&do64, dO, ntok, d, d, 64);
  if (!ok) return 1;
  const float scale = 1.f / sqrtf(float(HD));
  const float scale_log2 = scale * 1.4426950408889634f;
  const int nt = (T + 127) / 128;
  auto kq = attn_dq_tc_kernel<HD>;
  const int smem_q = int(DqSmem<HD>::BYTES);
  if (cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q) != cudaSuccess)
    return 1;
  kq<<<nt * B * H, kThreads, smem_q, st>>>(q128, do128, k64, v64,
                                           static_cast<const __nv_bfloat16*>(q), lse, Dbuf, rq,
                                           cos_t, sin_t, static_cast<__nv_bfloat16*>(dqkv), H, T,
                                           scale, scale_log2, c.qk_norm, status);
  auto kk = attn_dkv_tc_kernel<HD>;
  const int smem_k = int(DkvSmem<HD>::BYTES);
  if (cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_k) != cudaSuccess)
    return 1;
  kk<<<nt * B * H, kThreads, smem_k, st>>>(k128, v128, q64, do64,
                                           static_cast<const __nv_bfloat16*>(k), lse, Dbuf, rk,
                                           cos_t, sin_t, static_cast<__nv_bfloat16*>(dqkv), H, T,
                                           scale, scale_log2, c.qk_norm, status);
  return last_launch_rc();
}
}  // namespace

int launch_attn_bwd_tc(const gpt_config& c, const void* q, const void* k, const void* v,
                       const void* o, const void* dO, const float* lse, const float* rq,
                       const float* rk, const float* cos_t, const float* sin_t, float* Dbuf,
                       void* dqkv, int32_t* status, void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  return c.head_dim == 128
             ? attn_bwd_tc_t<128>(c, q, k, v, o, dO, lse, rq, rk, cos_t, sin_t, Dbuf, dqkv, status, st)
             : attn_bwd_tc_t<64>(c, q, k, v, o, dO, lse, rq, rk, cos_t, sin_t, Dbuf, dqkv, status, st);
}

}  // namespace gpt
