// Causal flash attention, forward and backward, on the sm_100a tensor cores.
//
// q, k, v: head-major [B*H*T, hd] bf16 (q and k already rotated and
// normalised); o, dO: token-major [B*T, H*hd] bf16; lse: [B*H*T] fp32, the
// log-sum-exp of each query row's scaled scores s_ij = q_i . k_j / sqrt(hd)
// over keys j <= i.
//
// Every kernel: warp 0 loads tiles with TMA (128-byte swizzle), one thread of
// warp 1 issues tcgen05.mma into tensor memory, warps 2..9 (256 threads, two
// per accumulator row: each TMEM lane quarter is read by two warps) do the
// element-wise work.  All mbarrier waits are bounded (GPT_ETIMEOUT in the
// status word); the compute warps reach their named barriers the same number
// of times on every path, so an expired wait cannot strand them.
#include <cudaTypedefs.h>

#include "device_common.cuh"
#include "tc_ptx.cuh"

namespace gpt {

namespace {
constexpr int BQ = 128, BKV = 128, kInner = 64;
constexpr int kThreads = 320;   // warp 0 TMA, warp 1 MMA, warps 2..9 compute
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;

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
// barrier among the 256 compute threads (warps 2..9)
__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// byte offset of 16-byte unit `u` (8 bf16) of row r of a [rows x 64] bf16 tile
// stored with the 128-byte swizzle (the layout TMA writes and the MMA reads)
__device__ __forceinline__ uint32_t sw_off(int r, int u) { return r * 128 + ((u ^ (r & 7)) << 4); }

struct Roles {
  int warp, lane, quarter, half, r;
  uint32_t lane_off;
};
__device__ __forceinline__ Roles roles() {
  Roles x;
  x.warp = threadIdx.x / 32;
  x.lane = threadIdx.x & 31;
  x.quarter = x.warp & 3;            // TMEM lanes 32*quarter .. +31
  x.half = (x.warp - 2) >> 2;        // compute warps 2..5 -> 0, 6..9 -> 1
  x.r = x.quarter * 32 + x.lane;     // accumulator row
  x.lane_off = uint32_t(x.quarter * 32) << 16;
  return x;
}

template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[N]) {
  static_assert(N == 16 || N == 32, "");
  uint32_t u[N];
  if constexpr (N == 32) tc::tmem_ld_32x32b_x32(taddr, u);
  else tc::tmem_ld_32x32b_x16(taddr, u);
  tc::tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < N; ++i) v[i] = __uint_as_float(u[i]);
}

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

// [rows, cols] bf16 row-major (pitch ld elements), box 64 columns x box_rows rows
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
}  // namespace

// Common prologue: barrier init by thread 0, TMEM allocation by warp 1.
#define ATTN_PROLOGUE(BARS, INIT)                 \
  if (threadIdx.x == 0) {                         \
    INIT;                                         \
    (BARS)->abort = 0;                            \
    tc::fence_barrier_init();                     \
  }                                               \
  if (threadIdx.x / 32 == 1) {                    \
    tc::tmem_alloc(&(BARS)->tmem_base, 512);      \
    tc::tmem_relinquish();                        \
  }                                               \
  tc::tc_fence_before();                          \
  __syncthreads();                                \
  tc::tc_fence_after();

#define ATTN_EPILOGUE(TMEM)                       \
  __syncwarp();                                   \
  tc::tc_fence_before();                          \
  __syncthreads();                                \
  if (threadIdx.x / 32 == 1) {                    \
    tc::tc_fence_after();                         \
    tc::tmem_dealloc((TMEM), 512);                \
  }

// ===========================================================================
// Forward.  One CTA per (128-query tile, b*h), the longest causal rows first.
// S_j = Q K_j^T into one of two TMEM score buffers; the compute threads (two
// per row, 64 keys each) take the row max (exchanged through shared memory),
// write P_j = 2^(s*log2e/sqrt(hd) - m) as bf16 into the swizzled P tile, and
// O += P_j V_j accumulates in TMEM.  A row's O and running sum are rescaled
// (tcgen05.ld/st, each thread its half of the columns) only when its max grows
// by more than 2^8 over the reference they share, so the result is exact and
// most tiles skip it.  K and V have separate 2-slot rings: K_{j+2} loads as soon
// as S_j is done, V_{j+2} once P_j V_j is.
// ===========================================================================
namespace {
template <int HD>
struct FwdSmem {
  static constexpr uint32_t TILE = BQ * HD * 2;
  static constexpr uint32_t P_BYTES = BQ * BKV * 2;
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t K_OFF = Q_OFF + TILE;
  static constexpr uint32_t V_OFF = K_OFF + 2 * TILE;
  static constexpr uint32_t P_OFF = V_OFF + 2 * TILE;
  static constexpr uint32_t RED_OFF = P_OFF + P_BYTES;           // float [2 iter][2 half][128]
  static constexpr uint32_t SUM_OFF = RED_OFF + 2 * 2 * BQ * 4;  // float [2 half][128]
  static constexpr uint32_t BAR_OFF = SUM_OFF + 2 * BQ * 4;
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;
  static_assert(K_OFF % 1024 == 0 && V_OFF % 1024 == 0 && P_OFF % 1024 == 0, "");
};
struct FwdBars {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2];
  uint64_t p_ready;
  uint64_t pv_full;
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};
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
  // (batch, head)-major order, longest causal rows first inside each head: the
  // CTAs resident together share a few heads' K/V, which then stay in L2
  const int n_qt = (T + BQ - 1) / BQ;
  const int bh = int(blockIdx.x) / n_qt;
  const int qt = n_qt - 1 - int(blockIdx.x) % n_qt;
  const int q0 = qt * BQ;
  const int n_kv = qt + 1;
  const int row_base = bh * T;
  constexpr uint32_t CH = BQ * 128;  // bytes of one 64-column chunk of a 128-row tile
  constexpr int NCH = HD / 64;

  ATTN_PROLOGUE(bars, {
    tc::mbar_init(&bars->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->k_full[s], 1); tc::mbar_init(&bars->k_empty[s], 1);
      tc::mbar_init(&bars->v_full[s], 1); tc::mbar_init(&bars->v_empty[s], 1);
      tc::mbar_init(&bars->s_full[s], 1);
    }
    tc::mbar_init(&bars->p_ready, 256);
    tc::mbar_init(&bars->pv_full, 1);
    tc::mbar_init(&bars->done, 1);
  })
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  const uint32_t t_o = tmem + 256;  // S buffers at columns 0 and 128

  if (warp == 0) {
    // lane 0: Q then the K ring; lane 1: the V ring
    if (lane < 2) {
      const bool is_k = lane == 0;
      uint64_t* full = is_k ? bars->k_full : bars->v_full;
      uint64_t* empty = is_k ? bars->k_empty : bars->v_empty;
      const CUtensorMap* map = is_k ? &map_k : &map_v;
      uint8_t* base = smem + (is_k ? S::K_OFF : S::V_OFF);
      uint32_t issued = 0, last_par = 0;
      if (is_k) {
        tc::mbar_arrive_expect_tx(&bars->q_full, S::TILE);
#pragma unroll
        for (int c = 0; c < NCH; ++c)
          tc::tma_load_2d(smem + S::Q_OFF + c * CH, &map_q, &bars->q_full, c * 64, row_base + q0);
      }
      for (int j = 0; j < n_kv; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!tc::mbar_wait_bounded(&empty[st], ph ^ 1, abort, kWaitNs)) {
          record_status(status, GPT_ETIMEOUT, K_ATTN, 10);
          *abort = 1;
          break;
        }
        tc::mbar_arrive_expect_tx(&full[st], S::TILE);
#pragma unroll
        for (int c = 0; c < NCH; ++c)
          tc::tma_load_2d(base + st * S::TILE + c * CH, map, &full[st], c * 64, row_base + j * BKV);
        issued |= 1u << st;
        last_par = (last_par & ~(1u << st)) | (ph << st);
      }
      if (*abort) {
        if (is_k) tc::mbar_wait_bounded(&bars->q_full, 0, nullptr, kWaitNs);
        for (int s = 0; s < 2; ++s)
          if (issued >> s & 1) tc::mbar_wait_bounded(&full[s], (last_par >> s) & 1, nullptr, kWaitNs);
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
        if (!tc::mbar_wait_bounded(&bars->v_full[j & 1], (j >> 1) & 1, abort, kWaitNs)) return false;
        tc::tc_fence_after();
        const uint32_t v_addr = tc::smem_u32(smem + S::V_OFF + (j & 1) * S::TILE);
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k)
          tc::mma_bf16_ss(t_o, tc::smem_desc_sw128(p_addr + (k >> 2) * CH + (k & 3) * 32, 16),
                          tc::smem_desc_sw128(v_addr + k * 2048, CH), idesc_pv, (j | k) != 0);
        tc::mma_commit(&bars->pv_full);
        tc::mma_commit(&bars->v_empty[j & 1]);
        return true;
      };
      for (int j = 0; ok && j < n_kv; ++j) {
        const int st = j & 1;
        if (!tc::mbar_wait_bounded(&bars->k_full[st], (j >> 1) & 1, abort, kWaitNs)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t k_addr = tc::smem_u32(smem + S::K_OFF + st * S::TILE);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t off = (k >> 2) * CH + (k & 3) * 32;
          tc::mma_bf16_ss(tmem + st * 128, tc::smem_desc_sw128(q_addr + off, 16),
                          tc::smem_desc_sw128(k_addr + off, 16), idesc_s, k != 0);
        }
        issued_any = true;
        tc::mma_commit(&bars->s_full[st]);
        tc::mma_commit(&bars->k_empty[st]);
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
    const Roles R = roles();
    const int q = q0 + R.r;
    float* red = reinterpret_cast<float*>(smem + S::RED_OFF);
    float* sums = reinterpret_cast<float*>(smem + S::SUM_OFF);
    uint8_t* p_chunk = smem + S::P_OFF + R.half * CH;  // this thread's 64 keys
    float m_ref = -INFINITY, l_half = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int st = j & 1;
      const int k0 = j * BKV + R.half * 64;
      if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->s_full[st], (j >> 1) & 1, abort, kWaitNs));
      float s[64];
      float mx = -INFINITY;
      if (ok) {
        tc::tc_fence_after();
        uint32_t ua[32], ub[32];
        tc::tmem_ld_32x32b_x32(tmem + st * 128 + R.lane_off + R.half * 64, ua);
        tc::tmem_ld_32x32b_x32(tmem + st * 128 + R.lane_off + R.half * 64 + 32, ub);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) { s[i] = __uint_as_float(ua[i]); s[32 + i] = __uint_as_float(ub[i]); }
        if (j == qt || k0 + 64 > T) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (k0 + i > q || k0 + i >= T) s[i] = -INFINITY;
        }
#pragma unroll
        for (int i = 0; i < 64; ++i) mx = fmaxf(mx, s[i]);
      }
      // row max over both halves (scores are unscaled here; the scale is positive)
      red[(st * 2 + R.half) * BQ + R.r] = mx;
      compute_bar();
      const float mx_all = fmaxf(red[(st * 2) * BQ + R.r], red[(st * 2 + 1) * BQ + R.r]) * scale_log2;
      if (ok && j > 0) {
        ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->pv_full, (j - 1) & 1, abort, kWaitNs));
        if (ok) tc::tc_fence_after();
      }
      if (ok) {
        const bool grow = mx_all > m_ref + 8.f;
        const float factor = grow ? ex2(m_ref - mx_all) : 1.f;
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int c = 0; c < HD / 2; c += 16) {
            uint32_t u[16];
            const uint32_t ta = t_o + R.lane_off + R.half * (HD / 2) + c;
            tc::tmem_ld_32x32b_x16(ta, u);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * factor);
            tc::tmem_st_32x32b_x16(ta, u);
          }
          tc::tmem_wait_st();
        }
        if (grow) {
          l_half *= factor;
          m_ref = mx_all;
        }
        float lsum = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = ex2(fmaf(s[u * 8 + 2 * e], scale_log2, -m_ref));
            const float p1 = ex2(fmaf(s[u * 8 + 2 * e + 1], scale_log2, -m_ref));
            lsum += p0 + p1;
            pk[e] = pack2(p0, p1);
          }
          *reinterpret_cast<uint4*>(p_chunk + sw_off(R.r, u)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        l_half += lsum;
        fence_async_smem();
        tc::tc_fence_before();
      }
      tc::mbar_arrive(&bars->p_ready);
    }
    if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->pv_full, (n_kv - 1) & 1, abort, kWaitNs));
    sums[R.half * BQ + R.r] = l_half;
    compute_bar();
    const float l = sums[R.r] + sums[BQ + R.r];
    if (!ok) {
      if (R.lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 12);
      *abort = 1;
    } else {
      tc::tc_fence_after();
      const int b = bh / H, h = bh % H;
      const float inv = 1.f / l;
      __nv_bfloat16* dst = o + (int64_t(b) * T + q) * (int64_t(H) * HD) + h * HD + R.half * (HD / 2);
#pragma unroll
      for (int c = 0; c < HD / 2; c += 32) {
        float v[32];
        tmem_ld<32>(t_o + R.lane_off + R.half * (HD / 2) + c, v);
        if (q < T) {
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            *reinterpret_cast<uint4*>(dst + c + i) =
                make_uint4(pack2(v[i] * inv, v[i + 1] * inv), pack2(v[i + 2] * inv, v[i + 3] * inv),
                           pack2(v[i + 4] * inv, v[i + 5] * inv), pack2(v[i + 6] * inv, v[i + 7] * inv));
        }
      }
      if (q < T && R.half == 0) lse[int64_t(bh) * T + q] = (m_ref + __log2f(l)) * 0.69314718055994531f;
    }
  }
  ATTN_EPILOGUE(tmem)
}

namespace {
template <int HD>
int attn_fwd_tc_t(const gpt_config& c, const void* q, const void* k, const void* v, void* o,
                  float* lse, int32_t* status, cudaStream_t st) {
  const uint64_t rows = uint64_t(c.batch) * c.n_head * c.seq_len;
  CUtensorMap mq, mk, mv;
  if (!tile_map(&mq, q, rows, HD, HD, 128) || !tile_map(&mk, k, rows, HD, HD, 128) ||
      !tile_map(&mv, v, rows, HD, HD, 128))
    return 1;
  auto kern = attn_fwd_tc_kernel<HD>;
  const int smem = int(FwdSmem<HD>::BYTES);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 1;
  const int n_qt = (c.seq_len + BQ - 1) / BQ;
  kern<<<n_qt * c.batch * c.n_head, kThreads, smem, st>>>(
      mq, mk, mv, static_cast<__nv_bfloat16*>(o), lse, c.n_head, c.seq_len,
      kLog2e / sqrtf(float(HD)), status);
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
// Backward.  With P_ij = exp(s_ij - lse_i) and D_i = dO_i . o_i:
//   dS_ij = P_ij (dO_i . v_j - D_i)
//   dQ_i  = sum_j dS_ij k_j / sqrt(hd)      (attn_dq_tc: CTA = 128 queries)
//   dK_j  = sum_i dS_ij q_i / sqrt(hd)      (attn_dkv_tc: CTA = 128 keys)
//   dV_j  = sum_i P_ij dO_i
// Each kernel owns its outputs, so no sum needs atomics (deterministic).  The
// gradients of q and k then go back through the per-head RMSNorm,
// dx = r (g - y mean(g y)), and the transposed RoPE rotation, and land in the
// [q | k | v] gradient rows [B*T, 3*H*hd].
// ===========================================================================
namespace {

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

constexpr int kRing = 3;    // slots of the per-step operand ring (dK/dV kernel)
constexpr int kRingQ = 4;   // slots of the K/V ring of the dQ kernel

struct BwdBars {
  uint64_t fixed_full;
  uint64_t ring_full[kRingQ];
  uint64_t ring_empty[kRingQ];
  uint64_t s_full[2];
  uint64_t ds_ready[2];
  uint64_t acc_full;
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

// One row's gradient w.r.t. its normalised, rotated q or k (TMEM, fp32, HD
// columns at `taddr`, times `scale`) back through RMSNorm (y: the normalised
// row, rr: its 1/rms) and RoPE, written as bf16.  The row's two compute
// threads split the rotation pairs: thread `half` takes pairs i in
// [half*HD/4, (half+1)*HD/4) and their partners i + HD/2; the mean(g y) of the
// norm is summed across both through `red` (one compute_bar, reached on every
// path).
template <int HD>
__device__ __forceinline__ void norm_rope_bwd_half(uint32_t taddr, int half, int r, float scale,
                                                   const __nv_bfloat16* __restrict__ y,
                                                   float rr, int qk_norm,
                                                   const float* __restrict__ cosr,
                                                   const float* __restrict__ sinr,
                                                   __nv_bfloat16* __restrict__ out, bool ok,
                                                   bool write, float* red) {
  constexpr int HALF = HD / 2, Q4 = HD / 4;
  const int i0 = half * Q4;
  float ga[Q4], gb[Q4], ya[Q4], yb[Q4];
  float part = 0.f;
  if (ok) {
#pragma unroll
    for (int c = 0; c < Q4; c += 16) {
      float ta[16], tb[16];
      tmem_ld<16>(taddr + i0 + c, ta);
      tmem_ld<16>(taddr + HALF + i0 + c, tb);
#pragma unroll
      for (int e = 0; e < 16; ++e) { ga[c + e] = ta[e] * scale; gb[c + e] = tb[e] * scale; }
    }
    if (write) {
#pragma unroll
      for (int c = 0; c < Q4; c += 8) {
        const uint4 ua = *reinterpret_cast<const uint4*>(y + i0 + c);
        const uint4 ub = *reinterpret_cast<const uint4*>(y + HALF + i0 + c);
        const uint32_t wa[4] = {ua.x, ua.y, ua.z, ua.w}, wb[4] = {ub.x, ub.y, ub.z, ub.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wa[e]));
          float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wb[e]));
          ya[c + 2 * e] = fa.x; ya[c + 2 * e + 1] = fa.y;
          yb[c + 2 * e] = fb.x; yb[c + 2 * e + 1] = fb.y;
        }
      }
#pragma unroll
      for (int i = 0; i < Q4; ++i) part += ga[i] * ya[i] + gb[i] * yb[i];
    }
  }
  red[half * 128 + r] = part;
  compute_bar();
  const float mean_gy = (red[r] + red[128 + r]) / float(HD);
  if (!ok || !write) return;
  uint32_t pa[Q4 / 2], pb[Q4 / 2];
#pragma unroll
  for (int i = 0; i < Q4; i += 2) {
    float a0 = ga[i], a1 = ga[i + 1], b0 = gb[i], b1 = gb[i + 1];
    if (qk_norm) {
      a0 = rr * (a0 - ya[i] * mean_gy); a1 = rr * (a1 - ya[i + 1] * mean_gy);
      b0 = rr * (b0 - yb[i] * mean_gy); b1 = rr * (b1 - yb[i + 1] * mean_gy);
    }
    const float c0 = cosr[i0 + i], s0 = sinr[i0 + i], c1 = cosr[i0 + i + 1], s1 = sinr[i0 + i + 1];
    pa[i / 2] = pack2(a0 * c0 + b0 * s0, a1 * c1 + b1 * s1);
    pb[i / 2] = pack2(-a0 * s0 + b0 * c0, -a1 * s1 + b1 * c1);
  }
#pragma unroll
  for (int i = 0; i < Q4 / 2; i += 4) {
    *reinterpret_cast<uint4*>(out + i0 + 2 * i) = make_uint4(pa[i], pa[i + 1], pa[i + 2], pa[i + 3]);
    *reinterpret_cast<uint4*>(out + HALF + i0 + 2 * i) = make_uint4(pb[i], pb[i + 1], pb[i + 2], pb[i + 3]);
  }
}

template <int HD>
struct DqSmem {
  static constexpr uint32_t BIG = 128 * HD * 2;
  static constexpr uint32_t SMALL = kInner * HD * 2;
  static constexpr uint32_t DS = 128 * kInner * 2;
  static constexpr uint32_t Q_OFF = 0, DO_OFF = BIG, K_OFF = 2 * BIG;
  static constexpr uint32_t V_OFF = K_OFF + kRingQ * SMALL;
  static constexpr uint32_t DS_OFF = V_OFF + kRingQ * SMALL;
  static constexpr uint32_t RED_OFF = DS_OFF + 2 * DS;
  static constexpr uint32_t BAR_OFF = RED_OFF + 2 * 128 * 4;
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;
  static_assert(K_OFF % 1024 == 0 && V_OFF % 1024 == 0 && DS_OFF % 1024 == 0, "");
};

}  // namespace

// dQ for 128 queries of one (batch, head), looping over 64-key tiles.  Compute
// thread (row, half) handles keys [32*half, 32*half + 32) of each tile.
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
  const int bh = int(blockIdx.x) / n_qt;  // (batch, head)-major, as in the forward
  const int qt = n_qt - 1 - int(blockIdx.x) % n_qt;
  const int b = bh / H, h = bh % H;
  const int q0 = qt * 128;
  const int n_steps = (min(q0 + 128, T) + kInner - 1) / kInner;
  constexpr int NCH = HD / 64;

  ATTN_PROLOGUE(bars, {
    tc::mbar_init(&bars->fixed_full, 1);
    for (int s = 0; s < kRingQ; ++s) {
      tc::mbar_init(&bars->ring_full[s], 1);
      tc::mbar_init(&bars->ring_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->ds_ready[s], 256);
    }
    tc::mbar_init(&bars->acc_full, 1);
    tc::mbar_init(&bars->done, 1);
  })
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  const uint32_t t_dq = tmem + 256;  // S/dP pairs at columns 0 and 128 (64 + 64 each)

  if (warp == 0) {
    if (lane == 0) {
      uint32_t issued = 0, last_par = 0;
      tc::mbar_arrive_expect_tx(&bars->fixed_full, 2 * S::BIG);
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        tc::tma_load_2d(smem + S::Q_OFF + c * (128 * 128), &map_q128, &bars->fixed_full, c * 64, bh * T + q0);
        tc::tma_load_2d(smem + S::DO_OFF + c * (128 * 128), &map_do128, &bars->fixed_full,
                        h * HD + c * 64, b * T + q0);
      }
      for (int j = 0; j < n_steps; ++j) {
        const int st = j % kRingQ;
        const uint32_t ph = (j / kRingQ) & 1;
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
        for (int s = 0; s < kRingQ; ++s)
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
        const uint32_t k_addr = tc::smem_u32(smem + S::K_OFF + (j % kRingQ) * S::SMALL);
#pragma unroll
        for (int k = 0; k < kInner / 16; ++k)
          tc::mma_bf16_ss(t_dq, tc::smem_desc_sw128(ds_addr + k * 32, 16),
                          tc::smem_desc_sw128(k_addr + k * 2048, kInner * 128), idesc_dq, (j | k) != 0);
        tc::mma_commit(&bars->ring_empty[j % kRingQ]);
        return true;
      };
      for (int j = 0; ok && j < n_steps; ++j) {
        const int st = j % kRingQ;
        if (!tc::mbar_wait_bounded(&bars->ring_full[st], (j / kRingQ) & 1, abort, kWaitNs)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t k_addr = tc::smem_u32(smem + S::K_OFF + st * S::SMALL);
        const uint32_t v_addr = tc::smem_u32(smem + S::V_OFF + st * S::SMALL);
        const uint32_t pair = tmem + (j & 1) * 128;
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t big = (k >> 2) * (128 * 128) + (k & 3) * 32;
          const uint32_t small = (k >> 2) * (kInner * 128) + (k & 3) * 32;
          tc::mma_bf16_ss(pair, tc::smem_desc_sw128(q_addr + big, 16),
                          tc::smem_desc_sw128(k_addr + small, 16), idesc_s, k != 0);
          tc::mma_bf16_ss(pair + kInner, tc::smem_desc_sw128(do_addr + big, 16),
                          tc::smem_desc_sw128(v_addr + small, 16), idesc_s, k != 0);
        }
        issued_any = true;
        tc::mma_commit(&bars->s_full[j & 1]);
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
    const Roles R = roles();
    const int q = q0 + R.r;
    const bool qv = q < T;
    const float lse2 = qv ? lse[int64_t(bh) * T + q] * kLog2e : 0.f;
    const float Dq = qv ? D[int64_t(bh) * T + q] : 0.f;
    bool ok = true;
    for (int j = 0; j < n_steps; ++j) {
      const int sb = j & 1;
      if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->s_full[sb], (j >> 1) & 1, abort, kWaitNs));
      if (ok) {
        tc::tc_fence_after();
        const int k0 = j * kInner + R.half * 32;
        uint32_t us[32], up[32];
        tc::tmem_ld_32x32b_x32(tmem + sb * 128 + R.lane_off + R.half * 32, us);
        tc::tmem_ld_32x32b_x32(tmem + sb * 128 + kInner + R.lane_off + R.half * 32, up);
        tc::tmem_wait_ld();
        const bool need_mask = !qv || k0 + 32 > q || k0 + 32 > T;
        uint8_t* rowp = smem + S::DS_OFF + sb * S::DS;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = u * 8 + 2 * e;
            float p0 = ex2(fmaf(__uint_as_float(us[i]), scale_log2, -lse2));
            float p1 = ex2(fmaf(__uint_as_float(us[i + 1]), scale_log2, -lse2));
            if (need_mask) {
              if (k0 + i > q || k0 + i >= T || !qv) p0 = 0.f;
              if (k0 + i + 1 > q || k0 + i + 1 >= T || !qv) p1 = 0.f;
            }
            pk[e] = pack2(p0 * (__uint_as_float(up[i]) - Dq), p1 * (__uint_as_float(up[i + 1]) - Dq));
          }
          *reinterpret_cast<uint4*>(rowp + sw_off(R.r, R.half * 4 + u)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        fence_async_smem();
        tc::tc_fence_before();
      }
      tc::mbar_arrive(&bars->ds_ready[sb]);
    }
    if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->acc_full, 0, abort, kWaitNs));
    if (!ok) {
      if (R.lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 22);
      *abort = 1;
    } else {
      tc::tc_fence_after();
    }
    const int d = H * HD;
    const int tq = qv ? q : 0;
    norm_rope_bwd_half<HD>(t_dq + R.lane_off, R.half, R.r, scale, qn + (int64_t(bh) * T + tq) * HD,
                           qv ? rq[int64_t(bh) * T + q] : 0.f, qk_norm, cos_t + tq * (HD / 2),
                           sin_t + tq * (HD / 2), dqkv + (int64_t(b) * T + tq) * 3 * d + h * HD, ok,
                           qv, reinterpret_cast<float*>(smem + S::RED_OFF));
  }
  ATTN_EPILOGUE(tmem)
}

namespace {
template <int HD>
struct DkvSmem {
  static constexpr uint32_t BIG = 128 * HD * 2;
  static constexpr uint32_t SMALL = kInner * HD * 2;
  static constexpr uint32_t PT = 128 * kInner * 2;
  static constexpr uint32_t K_OFF = 0, V_OFF = BIG, Q_OFF = 2 * BIG;
  static constexpr uint32_t DO_OFF = Q_OFF + kRing * SMALL;
  // swizzled tiles first: each must start on a 1024-byte boundary
  static constexpr uint32_t P_OFF = DO_OFF + kRing * SMALL;
  static constexpr uint32_t DS_OFF = P_OFF + 2 * PT;
  static constexpr uint32_t STAT_OFF = DS_OFF + 2 * PT;  // [ring][lse2 x 64 | D x 64]
  static constexpr uint32_t RED_OFF = P_OFF;  // epilogue only, after the last P is consumed
  static constexpr uint32_t BAR_OFF = STAT_OFF + kRing * 2 * kInner * 4;
  static_assert(P_OFF % 1024 == 0 && DS_OFF % 1024 == 0 && DO_OFF % 1024 == 0, "");
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;
};
}  // namespace

// dK, dV for 128 keys of one (batch, head), looping over 64-query tiles.
// Compute thread (key row, half) handles queries [32*half, 32*half + 32) of
// each tile; the producer warp stages lse and D of the tile's queries in
// shared memory next to the Q / dO tiles.
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
  const int bh = int(blockIdx.x) / n_kt;  // (batch, head)-major; key tile 0 (most queries) first
  const int kt = int(blockIdx.x) % n_kt;
  const int b = bh / H, h = bh % H;
  const int k0 = kt * 128;
  const int i_begin = k0 / kInner;
  const int n_steps = (T + kInner - 1) / kInner - i_begin;
  constexpr int NCH = HD / 64;

  ATTN_PROLOGUE(bars, {
    tc::mbar_init(&bars->fixed_full, 1);
    for (int s = 0; s < kRing; ++s) {
      tc::mbar_init(&bars->ring_full[s], 1 + 32);  // TMA bytes + the producer warp's stat stores
      tc::mbar_init(&bars->ring_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->ds_ready[s], 256);
    }
    tc::mbar_init(&bars->acc_full, 1);
    tc::mbar_init(&bars->done, 1);
  })
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  const uint32_t t_dv = tmem + 256, t_dk = tmem + 256 + HD;

  if (warp == 0) {
    uint32_t issued = 0, last_par = 0;
    if (lane == 0) {
      tc::mbar_arrive_expect_tx(&bars->fixed_full, 2 * S::BIG);
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        tc::tma_load_2d(smem + S::K_OFF + c * (128 * 128), &map_k128, &bars->fixed_full, c * 64, bh * T + k0);
        tc::tma_load_2d(smem + S::V_OFF + c * (128 * 128), &map_v128, &bars->fixed_full, c * 64, bh * T + k0);
      }
    }
    for (int j = 0; j < n_steps; ++j) {
      const int st = j % kRing;
      const uint32_t ph = (j / kRing) & 1;
      const int qs = (i_begin + j) * kInner;
      const bool ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->ring_empty[st], ph ^ 1, abort, kWaitNs));
      if (!ok) {
        if (lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 30);
        *abort = 1;
        break;
      }
      if (lane == 0) {
        tc::mbar_arrive_expect_tx(&bars->ring_full[st], 2 * S::SMALL);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          tc::tma_load_2d(smem + S::Q_OFF + st * S::SMALL + c * (kInner * 128), &map_q64,
                          &bars->ring_full[st], c * 64, bh * T + qs);
          tc::tma_load_2d(smem + S::DO_OFF + st * S::SMALL + c * (kInner * 128), &map_do64,
                          &bars->ring_full[st], h * HD + c * 64, b * T + qs);
        }
      }
      float* stat = reinterpret_cast<float*>(smem + S::STAT_OFF) + st * 2 * kInner;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int qi = lane * 2 + e;
        const int qq = qs + qi;
        stat[qi] = qq < T ? lse[int64_t(bh) * T + qq] * kLog2e : 0.f;
        stat[kInner + qi] = qq < T ? D[int64_t(bh) * T + qq] : 0.f;
      }
      tc::mbar_arrive(&bars->ring_full[st]);
      issued |= 1u << st;
      last_par = (last_par & ~(1u << st)) | (ph << st);
    }
    if (lane == 0 && *abort) {
      tc::mbar_wait_bounded(&bars->fixed_full, 0, nullptr, kWaitNs);
      for (int s = 0; s < kRing; ++s)
        if (issued >> s & 1) tc::mbar_wait_bounded(&bars->ring_full[s], (last_par >> s) & 1, nullptr, kWaitNs);
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
        const uint32_t q_addr = tc::smem_u32(smem + S::Q_OFF + (j % kRing) * S::SMALL);
        const uint32_t do_addr = tc::smem_u32(smem + S::DO_OFF + (j % kRing) * S::SMALL);
#pragma unroll
        for (int k = 0; k < kInner / 16; ++k) {
          tc::mma_bf16_ss(t_dv, tc::smem_desc_sw128(p_addr + k * 32, 16),
                          tc::smem_desc_sw128(do_addr + k * 2048, kInner * 128), idesc_acc, (j | k) != 0);
          tc::mma_bf16_ss(t_dk, tc::smem_desc_sw128(ds_addr + k * 32, 16),
                          tc::smem_desc_sw128(q_addr + k * 2048, kInner * 128), idesc_acc, (j | k) != 0);
        }
        tc::mma_commit(&bars->ring_empty[j % kRing]);
        return true;
      };
      for (int j = 0; ok && j < n_steps; ++j) {
        const int st = j % kRing;
        if (!tc::mbar_wait_bounded(&bars->ring_full[st], (j / kRing) & 1, abort, kWaitNs)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t q_addr = tc::smem_u32(smem + S::Q_OFF + st * S::SMALL);
        const uint32_t do_addr = tc::smem_u32(smem + S::DO_OFF + st * S::SMALL);
        const uint32_t pair = tmem + (j & 1) * 128;
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t big = (k >> 2) * (128 * 128) + (k & 3) * 32;
          const uint32_t small = (k >> 2) * (kInner * 128) + (k & 3) * 32;
          tc::mma_bf16_ss(pair, tc::smem_desc_sw128(k_addr + big, 16),
                          tc::smem_desc_sw128(q_addr + small, 16), idesc_s, k != 0);
          tc::mma_bf16_ss(pair + kInner, tc::smem_desc_sw128(v_addr + big, 16),
                          tc::smem_desc_sw128(do_addr + small, 16), idesc_s, k != 0);
        }
        issued_any = true;
        tc::mma_commit(&bars->s_full[j & 1]);
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
    const Roles R = roles();
    const int key = k0 + R.r;
    const bool kv = key < T;
    bool ok = true;
    for (int j = 0; j < n_steps; ++j) {
      const int sb = j & 1, st = j % kRing;
      // the producer warp stored this step's stats before arriving on
      // ring_full[st]; waiting on that phase makes them visible here
      if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->s_full[sb], (j >> 1) & 1, abort, kWaitNs));
      if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->ring_full[st], (j / kRing) & 1, abort, kWaitNs));
      if (ok) {
        tc::tc_fence_after();
        const int qs = (i_begin + j) * kInner + R.half * 32;
        const float* stat = reinterpret_cast<const float*>(smem + S::STAT_OFF) + st * 2 * kInner + R.half * 32;
        uint32_t us[32], up[32];
        tc::tmem_ld_32x32b_x32(tmem + sb * 128 + R.lane_off + R.half * 32, us);
        tc::tmem_ld_32x32b_x32(tmem + sb * 128 + kInner + R.lane_off + R.half * 32, up);
        tc::tmem_wait_ld();
        const bool need_mask = !kv || qs < key || qs + 32 > T;
        uint8_t* prow = smem + S::P_OFF + sb * S::PT;
        uint8_t* drow = smem + S::DS_OFF + sb * S::PT;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t pp[4], pd[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = u * 8 + 2 * e;
            float p0 = ex2(fmaf(__uint_as_float(us[i]), scale_log2, -stat[i]));
            float p1 = ex2(fmaf(__uint_as_float(us[i + 1]), scale_log2, -stat[i + 1]));
            if (need_mask) {
              if (qs + i < key || qs + i >= T || !kv) p0 = 0.f;
              if (qs + i + 1 < key || qs + i + 1 >= T || !kv) p1 = 0.f;
            }
            pp[e] = pack2(p0, p1);
            pd[e] = pack2(p0 * (__uint_as_float(up[i]) - stat[kInner + i]),
                          p1 * (__uint_as_float(up[i + 1]) - stat[kInner + i + 1]));
          }
          const uint32_t off = sw_off(R.r, R.half * 4 + u);
          *reinterpret_cast<uint4*>(prow + off) = make_uint4(pp[0], pp[1], pp[2], pp[3]);
          *reinterpret_cast<uint4*>(drow + off) = make_uint4(pd[0], pd[1], pd[2], pd[3]);
        }
        fence_async_smem();
        tc::tc_fence_before();
      }
      tc::mbar_arrive(&bars->ds_ready[sb]);
    }
    if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_bounded(&bars->acc_full, 0, abort, kWaitNs));
    if (!ok) {
      if (R.lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 32);
      *abort = 1;
    } else {
      tc::tc_fence_after();
    }
    const int d = H * HD;
    const int tk = kv ? key : 0;
    __nv_bfloat16* row = dqkv + (int64_t(b) * T + tk) * 3 * d;
    if (ok) {  // dV: this thread's half of the columns
#pragma unroll
      for (int c = 0; c < HD / 2; c += 32) {
        float v[32];
        tmem_ld<32>(t_dv + R.lane_off + R.half * (HD / 2) + c, v);
        if (kv) {
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            *reinterpret_cast<uint4*>(row + 2 * d + h * HD + R.half * (HD / 2) + c + i) =
                make_uint4(pack2(v[i], v[i + 1]), pack2(v[i + 2], v[i + 3]), pack2(v[i + 4], v[i + 5]),
                           pack2(v[i + 6], v[i + 7]));
        }
      }
    }
    norm_rope_bwd_half<HD>(t_dk + R.lane_off, R.half, R.r, scale, kn + (int64_t(bh) * T + tk) * HD,
                           kv ? rk[int64_t(bh) * T + key] : 0.f, qk_norm, cos_t + tk * (HD / 2),
                           sin_t + tk * (HD / 2), row + d + h * HD, ok, kv,
                           reinterpret_cast<float*>(smem + S::RED_OFF));
  }
  ATTN_EPILOGUE(tmem)
}

namespace {
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
  const float scale_log2 = scale * kLog2e;
  const int nt = (T + 127) / 128;
  auto kq = attn_dq_tc_kernel<HD>;
  const int smem_q = int(DqSmem<HD>::BYTES);
  if (cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q) != cudaSuccess)
    return 1;
  kq<<<nt * B * H, kThreads, smem_q, st>>>(q128, do128, k64, v64, static_cast<const __nv_bfloat16*>(q),
                                           lse, Dbuf, rq, cos_t, sin_t,
                                           static_cast<__nv_bfloat16*>(dqkv), H, T, scale,
                                           scale_log2, c.qk_norm, status);
  auto kk = attn_dkv_tc_kernel<HD>;
  const int smem_k = int(DkvSmem<HD>::BYTES);
  if (cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_k) != cudaSuccess)
    return 1;
  kk<<<nt * B * H, kThreads, smem_k, st>>>(k128, v128, q64, do64, static_cast<const __nv_bfloat16*>(k),
                                           lse, Dbuf, rk, cos_t, sin_t,
                                           static_cast<__nv_bfloat16*>(dqkv), H, T, scale,
                                           scale_log2, c.qk_norm, status);
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
