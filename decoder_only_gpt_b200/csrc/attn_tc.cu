// Causal flash attention, forward and backward, on the sm_100a tensor cores.
//
// q: head-major [B*H*T, hd] bf16, k, v: [B*Hkv*T, hd] (q and k already
// rotated and normalised; query head h reads key/value head h / (H/Hkv),
// grouped-query attention when Hkv < H); o, dO: token-major [B*T, H*hd] bf16;
// lse: [B*H*T] fp32, the log-sum-exp of each query row's scaled scores
// s_ij = q_i . k_j / sqrt(hd) over its visible keys i - W < j <= i (W, the
// sliding window, longer than any sequence when unset).  Each kernel visits
// only the key (or query) tiles that hold visible pairs and masks the rest
// inside the boundary tiles.
//
// Every kernel: warp 0 loads tiles with TMA (128-byte swizzle), warps 1 and 10
// issue tcgen05.mma into tensor memory (two independent MMA chains: one warp
// issues an MMA only every ~90 cycles, slower than the tensor pipe runs the
// small-N products of attention), warps 2..9 (256 threads, two per
// accumulator row: each TMEM lane quarter is read by two warps) do the
// element-wise work.  All mbarrier waits are bounded (GPT_ETIMEOUT in the
// status word); the compute warps reach their named barriers the same number
// of times on every path, so an expired wait cannot strand them.
#include <cudaTypedefs.h>

#include <algorithm>

#include "device_common.cuh"
#include "tc_ptx.cuh"

namespace gpt {

namespace {
constexpr int kThreads = 352;   // warp 0 TMA, warps 1 and 10 MMA, warps 2..9 compute
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
// Packed fp32 pairs (sm_100 f32x2 arithmetic: two IEEE fp32 operations per
// instruction, results identical to the scalar ones).
__device__ __forceinline__ uint64_t f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 unf2(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// barrier among the 256 compute threads (warps 2..9)
__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

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

// Work item of CTA `b` in a launch over n_rows x n_ranks items (a row is a
// (batch, head) and rank 0 its longest tile, the work shrinking with the
// rank): rows go in groups of kGroupRows, and inside a group all rows' rank-0
// items come first, then their rank-1 items, and so on.  The resident CTAs
// then share a few rows' K/V in L2, and the short items of the last group
// fill the tail instead of one row's long ones.
constexpr int kGroupRows = 16;
__device__ __forceinline__ void grouped_item(int b, int n_rows, int n_ranks, int& row, int& rank) {
  const int grp = b / (kGroupRows * n_ranks);
  const int base = grp * kGroupRows;
  const int gs = min(kGroupRows, n_rows - base);
  const int r = b - grp * kGroupRows * n_ranks;
  rank = r / gs;
  row = base + r % gs;
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
// The [B, T, ld] bf16 rows of the q|k|v gradient as a 3-D map with boxes of 64
// columns x 128 positions x 1 sequence: a box past position T - 1 is clipped
// at the end of its own sequence.
bool seq_map(CUtensorMap* m, const void* base, uint64_t B, uint64_t T, uint64_t ld) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {ld, T, B};
  cuuint64_t strides[2] = {ld * 2, T * ld * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// [rows, cols] fp32 row-major (pitch ld elements), box 32 columns x box_rows rows
bool tile_map_f32(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                  uint32_t box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 4};
  cuuint32_t box[2] = {32, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
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
// Forward.  A persistent grid (one CTA per SM) takes work items from a
// counter: an item is a pair of consecutive 128-query tiles (A = 2p, B = 2p+1)
// of one (batch, head), which share one stream of K and V tiles.  Items go in
// groups of heads, the longest pairs first (grouped_item), so the resident
// CTAs share a few heads' K/V in L2 and the short items fill the tail.
//
// Warps 0..3 own tile A's rows and warps 4..7 tile B's (one thread per query
// row: TMEM lane quarter = warp % 4); warp 8 publishes the items and loads
// tiles with TMA; warp 9 issues S_X = Q_X K^T and O_X += P_X V; warps 10 and
// 11 only complete their warpgroup.  TMEM: S_A at columns 0..127, S_B at
// 128..255, O_A at 256, O_B at 384.  A row's thread reads its 128 scores and
// writes P = 2^(s*log2e/sqrt(hd) - m) as packed bf16 over the first 64
// columns of its own S (the A operand of the PV product, read from TMEM), so
// the two tiles alternate on the tensor core: while one tile's exponentials
// run, the other tile's products do.  S_X of the next key tile overwrites
// P_X; it is issued after the PV product that reads P_X, by the same thread,
// so in order.  A row rescales its O and running sum (tcgen05.ld/st) only
// when its max grows by more than 2^8 over the reference they share: exact,
// and rare after the first tiles.  K_j and V_j take consecutive slots of one
// 4-slot ring.
// ===========================================================================
namespace {
constexpr int kFwdRing = 4;
constexpr int kFwdThreads = 384;  // warps 0..7 softmax, 8 TMA, 9 MMA, 10..11 idle
// Register split between the warpgroups (setmaxnreg): the launch gives every
// thread 168 (65,536 / 384 rounded down to the allocation granule of 8, and
// 3 x 168 x 32 fits one sub-partition's 16K); warpgroup 2 (TMA, MMA) gives
// registers back so that the two softmax warpgroups can each hold a row's 128
// scores.  2 x 128 x 200 + 128 x 104 = 64,512 = 384 x 168: the raise never
// waits for registers that are not there.
constexpr int kFwdRegsSoftmax = 200, kFwdRegsOther = 104;
static_assert(2 * 128 * kFwdRegsSoftmax + 128 * kFwdRegsOther <= kFwdThreads * 168, "");

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int HD>
struct FwdSmem {
  static constexpr uint32_t TILE = 128 * HD * 2;  // a 128-row Q, K or V tile
  static constexpr uint32_t QA_OFF = 0, QB_OFF = TILE;
  static constexpr uint32_t RING_OFF = 2 * TILE;
  static constexpr uint32_t BAR_OFF = RING_OFF + kFwdRing * TILE;
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;
  static_assert(TILE % 1024 == 0 && BYTES <= 232448, "");
};
struct FwdBars {
  uint64_t q_full[2], q_empty[2];
  uint64_t kv_full[kFwdRing], kv_empty[kFwdRing];
  uint64_t s_full[2], p_ready[2], pv_done[2];
  uint64_t item_full[2], item_empty[2];
  uint64_t done_s;
  uint32_t tmem_base;
  int abort;
  int items[2];  // the published work items (-1: none left)
};

// Key-tile range [lo, lo + n) of query tile qt (n = 0: the tile is past T).
struct KeyRange {
  int lo, n;
};
__device__ __forceinline__ KeyRange key_range(int qt, int T, int W) {
  KeyRange r;
  const int q0 = qt * 128;
  r.lo = max(0, q0 - W + 1) / 128;
  r.n = q0 < T ? qt - r.lo + 1 : 0;
  return r;
}
}  // namespace

// Work counters of the persistent kernels, in the unused tail of the
// workspace's 256-byte status region (which gpt_forward_loss zeroes): a pair
// per kernel, [next item, CTAs finished].  The last CTA of a launch to finish
// sets both back to zero, so every launch starts from zero without a memset.
constexpr int kSchedFwd = 0;
__host__ __device__ inline int32_t* sched_counters(int32_t* status, int which) {
  return status + 32 + which;  // bytes 128.. of the status region
}
__device__ __forceinline__ void sched_finish(int32_t* sched) {
  __threadfence();
  if (atomicAdd(sched + 1, 1) == int(gridDim.x) - 1) {
    atomicExch(sched, 0);
    atomicExch(sched + 1, 0);
  }
}

template <int HD>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                       const __grid_constant__ CUtensorMap map_k,
                       const __grid_constant__ CUtensorMap map_v, __nv_bfloat16* __restrict__ o,
                       float* __restrict__ lse, int H, int Hkv, int T, int W, float scale_log2,
                       int n_rows, int32_t* status) {
  using S = FwdSmem<HD>;
  constexpr int NCH = HD / 64;
  constexpr uint32_t CH = 128 * 128;  // bytes of one 64-column chunk of a 128-row tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + S::BAR_OFF);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int n_qt = (T + 127) / 128, n_pairs = (n_qt + 1) / 2;
  const int n_items = n_rows * n_pairs;
  int32_t* sched = sched_counters(status, kSchedFwd);

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(&bars->q_full[x], 1);
      tc::mbar_init(&bars->q_empty[x], 1);
      tc::mbar_init(&bars->s_full[x], 1);
      tc::mbar_init(&bars->p_ready[x], 128);
      tc::mbar_init(&bars->pv_done[x], 1);
      tc::mbar_init(&bars->item_full[x], 1);
      tc::mbar_init(&bars->item_empty[x], 9);  // the MMA warp and the 8 softmax warps
    }
    for (int s = 0; s < kFwdRing; ++s) {
      tc::mbar_init(&bars->kv_full[s], 1);
      tc::mbar_init(&bars->kv_empty[s], 1);
    }
    tc::mbar_init(&bars->done_s, 1);
    bars->abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 9) {
    tc::tmem_alloc(&bars->tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  volatile int* items = bars->items;
  // the item's (batch, head) row, query-tile pair and both tiles' key ranges
  auto decode = [=](int k, int& bh, int& pair, KeyRange& ra, KeyRange& rb) {
    int rank;
    grouped_item(k, n_rows, n_pairs, bh, rank);
    pair = n_pairs - 1 - rank;
    ra = key_range(2 * pair, T, W);
    rb = key_range(2 * pair + 1, T, W);
  };
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kFwdRegsOther));
  }
  if (warp == 8) {
    // TMA producer and scheduler: publishes each work item (-1 at the end),
    // then loads its Q tiles and its stream of K, V tiles
    if (lane == 0) {
      uint32_t ring_issued = 0, ring_par = 0, q_issued = 0, q_par = 0;
      int u = 0, qn[2] = {0, 0};
      bool ok = true;
      int k = int(blockIdx.x);
      for (int seq = 0;; ++seq) {
        const int s = seq & 1;
        if (!tc::mbar_wait_bounded(&bars->item_empty[s], ((seq >> 1) & 1) ^ 1, abort, kWaitNs)) { ok = false; break; }
        items[s] = k < n_items ? k : -1;
        tc::mbar_arrive(&bars->item_full[s]);
        if (k >= n_items) break;
        int bh, pair;
        KeyRange ra, rb;
        decode(k, bh, pair, ra, rb);
        const int n_kt = rb.n ? rb.lo + rb.n - ra.lo : ra.n;
        const int kv_row_base = ((bh / H) * Hkv + (bh % H) / (H / Hkv)) * T;
        for (int x = 0; ok && x < 2; ++x) {
          if ((x ? rb : ra).n == 0) continue;
          // the previous item's S products of this tile are done with Q_x
          if (!tc::mbar_wait_bounded(&bars->q_empty[x], (qn[x] & 1) ^ 1, abort, kWaitNs)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(&bars->q_full[x], S::TILE);
#pragma unroll
          for (int c = 0; c < NCH; ++c)
            tc::tma_load_2d(smem + (x ? S::QB_OFF : S::QA_OFF) + c * CH, &map_q, &bars->q_full[x], c * 64,
                            bh * T + (2 * pair + x) * 128);
          q_issued |= 1u << x;
          q_par = (q_par & ~(1u << x)) | ((qn[x] & 1u) << x);
          ++qn[x];
        }
        for (int v = 0; ok && v < 2 * n_kt; ++v, ++u) {  // K_j, V_j, K_j+1, ...
          const int st = u % kFwdRing;
          const uint32_t ph = (u / kFwdRing) & 1;
          if (!tc::mbar_wait_bounded(&bars->kv_empty[st], ph ^ 1, abort, kWaitNs)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(&bars->kv_full[st], S::TILE);
          const CUtensorMap* map = (v & 1) ? &map_v : &map_k;
#pragma unroll
          for (int c = 0; c < NCH; ++c)
            tc::tma_load_2d(smem + S::RING_OFF + st * S::TILE + c * CH, map, &bars->kv_full[st], c * 64,
                            kv_row_base + (ra.lo + v / 2) * 128);
          ring_issued |= 1u << st;
          ring_par = (ring_par & ~(1u << st)) | (ph << st);
        }
        if (!ok) break;
        k = atomicAdd(sched, 1) + int(gridDim.x);
      }
      if (!ok) {
        record_status(status, GPT_ETIMEOUT, K_ATTN, 10);
        *abort = 1;
        // wait for this warp's own copies in flight before the CTA exits
        for (int x = 0; x < 2; ++x)
          if (q_issued >> x & 1) tc::mbar_wait_bounded(&bars->q_full[x], (q_par >> x) & 1, nullptr, kWaitNs);
        for (int s = 0; s < kFwdRing; ++s)
          if (ring_issued >> s & 1) tc::mbar_wait_bounded(&bars->kv_full[s], (ring_par >> s) & 1, nullptr, kWaitNs);
      }
    }
  } else if (warp == 9) {
    // One warp issues every product, so they run in issue order.  Per key
    // tile j: O_A += P_A V_j as soon as tile A's threads have written P_A,
    // then at once S_A = Q_A K_{j+1}^T (over P_A's columns, after the product
    // that reads them), then the same for tile B.  A tile's next scores are
    // thus two products after its P, while the other tile's exponentials run.
    constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(128, HD, false, true);
    const uint32_t ring0 = tc::smem_u32(smem + S::RING_OFF);
    const uint32_t qa = tc::smem_u32(smem + S::QA_OFF), qb = tc::smem_u32(smem + S::QB_OFF);
    bool ok = true, issued_any = false;
    int u = 0, qn[2] = {0, 0}, cs[2] = {0, 0};  // ring items, Q fills, steps done per tile
    for (int seq = 0; ok; ++seq) {
      const int s = seq & 1;
      if (!tc::mbar_wait_warp(&bars->item_full[s], (seq >> 1) & 1, abort, kWaitNs)) { ok = false; break; }
      const int k = items[s];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->item_empty[s]);
      if (k < 0) break;
      int bh, pair;
      KeyRange ra, rb;
      decode(k, bh, pair, ra, rb);
      const int lo = ra.lo, n_kt = rb.n ? rb.lo + rb.n - ra.lo : ra.n;
      auto step_of = [=](int x, int j) {  // tile x's step at stream step j, or -1
        const KeyRange r = x ? rb : ra;
        const int i = lo + j - r.lo;
        return i >= 0 && i < r.n ? i : -1;
      };
      // S_X = Q_X K^T, the K tile in ring slot `st`; Q_X freed after its last
      auto issue_s = [&](int x, int st, bool last) {
        const uint64_t kd = tc::smem_desc_sw128(ring0 + st * S::TILE, 16);
        const uint64_t qd = tc::smem_desc_sw128(x ? qb : qa, 16);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * CH + (kk & 3) * 32;
          tc::mma_bf16_ss_elect(tmem + x * 128, tc::desc_advance(qd, off), tc::desc_advance(kd, off), idesc_s,
                                kk != 0);
        }
        tc::mma_commit_elect(&bars->s_full[x]);
        if (last) tc::mma_commit_elect(&bars->q_empty[x]);
      };
      for (int x = 0; ok && x < 2; ++x)
        if ((x ? rb : ra).n && !tc::mbar_wait_warp(&bars->q_full[x], qn[x]++ & 1, abort, kWaitNs)) ok = false;
      if (!ok) break;
      {
        const int st = u % kFwdRing;
        if (!tc::mbar_wait_warp(&bars->kv_full[st], (u / kFwdRing) & 1, abort, kWaitNs)) { ok = false; break; }
        tc::tc_fence_after();
        for (int x = 0; x < 2; ++x)
          if (step_of(x, 0) == 0) issue_s(x, st, (x ? rb : ra).n == 1);
        issued_any = true;
        tc::mma_commit_elect(&bars->kv_empty[st]);
      }
      for (int j = 0; ok && j < n_kt; ++j) {
        const int uv = u + 2 * j + 1, sv = uv % kFwdRing;
        const int uk = u + 2 * j + 2, sk = uk % kFwdRing;  // K of step j+1
        if (!tc::mbar_wait_warp(&bars->kv_full[sv], (uv / kFwdRing) & 1, abort, kWaitNs)) { ok = false; break; }
        const uint64_t vd = tc::smem_desc_sw128(ring0 + sv * S::TILE, CH);
        bool k_waited = false;
        for (int x = 0; ok && x < 2; ++x) {
          const int i = step_of(x, j);
          if (i >= 0) {
            if (!tc::mbar_wait_warp(&bars->p_ready[x], (cs[x] + i) & 1, abort, kWaitNs)) { ok = false; break; }
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk)
              tc::mma_bf16_ts_elect(tmem + 256 + x * 128, tmem + x * 128 + 8 * kk, tc::desc_advance(vd, kk * 2048),
                                    idesc_pv, (i | kk) != 0);
            tc::mma_commit_elect(&bars->pv_done[x]);
          }
          const int i1 = j + 1 < n_kt ? step_of(x, j + 1) : -1;
          if (i1 >= 0) {
            if (!k_waited) {
              if (!tc::mbar_wait_warp(&bars->kv_full[sk], (uk / kFwdRing) & 1, abort, kWaitNs)) { ok = false; break; }
              tc::tc_fence_after();
              k_waited = true;
            }
            issue_s(x, sk, i1 == (x ? rb : ra).n - 1);
          }
        }
        if (!ok) break;
        tc::mma_commit_elect(&bars->kv_empty[sv]);
        if (k_waited) tc::mma_commit_elect(&bars->kv_empty[sk]);
      }
      u += 2 * n_kt;
      cs[0] += ra.n;
      cs[1] += rb.n;
    }
    if (!ok) {
      if (lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 11);
      *abort = 1;
    }
    if (issued_any) {
      tc::mma_commit_elect(&bars->done_s);
      tc::mbar_wait_warp(&bars->done_s, 0, nullptr, kWaitNs);
    }
  } else if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kFwdRegsSoftmax));
    // softmax: thread = one query row of tile x
    const int x = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + x * 128 + lane_off, t_o = tmem + 256 + x * 128 + lane_off;
    bool ok = true;
    int cs = 0;  // this tile's steps done over the previous items
    for (int seq = 0; ok; ++seq) {
      const int s = seq & 1;
      if (!tc::mbar_wait_warp(&bars->item_full[s], (seq >> 1) & 1, abort, kWaitNs)) { ok = false; break; }
      const int k = items[s];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->item_empty[s]);
      if (k < 0) break;
      int bh, pair;
      KeyRange ra, rb;
      decode(k, bh, pair, ra, rb);
      const KeyRange r = x ? rb : ra;
      const int q = (2 * pair + x) * 128 + row;
      const int lo_key = q - W + 1;  // the row's first visible key
      float m_ref = -INFINITY, l = 0.f;
      for (int i = 0; ok && i < r.n; ++i) {
        const int k0 = (r.lo + i) * 128;
        if (!tc::mbar_wait_warp(&bars->s_full[x], (cs + i) & 1, abort, kWaitNs)) { ok = false; break; }
        tc::tc_fence_after();
        float sc[128];
        {
          uint32_t u0[32], u1[32], u2[32], u3[32];
          tc::tmem_ld_32x32b_x32(t_s, u0);
          tc::tmem_ld_32x32b_x32(t_s + 32, u1);
          tc::tmem_ld_32x32b_x32(t_s + 64, u2);
          tc::tmem_ld_32x32b_x32(t_s + 96, u3);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            sc[e] = __uint_as_float(u0[e]);
            sc[32 + e] = __uint_as_float(u1[e]);
            sc[64 + e] = __uint_as_float(u2[e]);
            sc[96 + e] = __uint_as_float(u3[e]);
          }
        }
        if (k0 + 127 > q || k0 + 128 > T || k0 < lo_key) {
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (k0 + e > q || k0 + e >= T || k0 + e < lo_key) sc[e] = -INFINITY;
        }
        float m4[4] = {sc[0], sc[1], sc[2], sc[3]};  // four independent chains
#pragma unroll
        for (int e = 4; e < 128; e += 8)
#pragma unroll
          for (int c = 0; c < 4; ++c) m4[c] = fmax3(m4[c], sc[e + 2 * c], sc[e + 2 * c + 1]);
        // scores are unscaled here; the scale is positive
        float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * scale_log2;
        const bool grow = mx > m_ref + 8.f;
        const float factor = grow ? ex2(m_ref - mx) : 1.f;
        if (grow) {
          l *= factor;
          m_ref = mx;
        }
        // a row whose keys so far were all outside its window has no reference
        // yet: its P is 0 (exp2(-inf - 0)), not NaN
        const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
        const uint64_t sc2 = f2(scale_log2, scale_log2), nm2 = f2(-m_use, -m_use);
        uint64_t lsum2[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float2 xx = unf2(fma2(f2(sc[64 * h + 2 * e], sc[64 * h + 2 * e + 1]), sc2, nm2));
            const float p0 = ex2(xx.x), p1 = ex2(xx.y);
            lsum2[e & 3] = add2(lsum2[e & 3], f2(p0, p1));
            pk[e] = pack2(p0, p1);
          }
          tc::tmem_st_32x32b_x32(t_s + 32 * h, pk);  // P over this row's first 64 S columns
        }
        const float2 ls = unf2(add2(add2(lsum2[0], lsum2[1]), add2(lsum2[2], lsum2[3])));
        l += ls.x + ls.y;
        if (i > 0 && __any_sync(0xffffffffu, grow)) {
          // O holds P V up to step i-1 once that product is done
          if (!tc::mbar_wait_warp(&bars->pv_done[x], (cs + i - 1) & 1, abort, kWaitNs)) { ok = false; break; }
          tc::tc_fence_after();
#pragma unroll
          for (int c = 0; c < HD; c += 32) {
            uint32_t uu[32];
            tc::tmem_ld_32x32b_x32(t_o + c, uu);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) uu[e] = __float_as_uint(__uint_as_float(uu[e]) * factor);
            tc::tmem_st_32x32b_x32(t_o + c, uu);
          }
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&bars->p_ready[x]);
      }
      if (!ok) break;
      if (r.n > 0) {
        if (!tc::mbar_wait_warp(&bars->pv_done[x], (cs + r.n - 1) & 1, abort, kWaitNs)) { ok = false; break; }
        tc::tc_fence_after();
        const int b = bh / H, h = bh % H;
        const float inv = 1.f / l;
        __nv_bfloat16* dst = o + (int64_t(b) * T + q) * (int64_t(H) * HD) + h * HD;
#pragma unroll
        for (int c = 0; c < HD; c += 32) {
          float v[32];
          tmem_ld<32>(t_o + c, v);
          if (q < T) {
#pragma unroll
            for (int e = 0; e < 32; e += 8)
              *reinterpret_cast<uint4*>(dst + c + e) =
                  make_uint4(pack2(v[e] * inv, v[e + 1] * inv), pack2(v[e + 2] * inv, v[e + 3] * inv),
                             pack2(v[e + 4] * inv, v[e + 5] * inv), pack2(v[e + 6] * inv, v[e + 7] * inv));
          }
        }
        if (q < T) lse[int64_t(bh) * T + q] = (m_ref + __log2f(l)) * 0.69314718055994531f;
        // the next item's first O_x += P_x V overwrites these columns only
        // after this warp's next p_ready arrival, which follows these reads
        tc::tc_fence_before();
      }
      cs += r.n;
    }
    if (!ok) {
      if (lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 12);
      *abort = 1;
    }
  }
  __syncwarp();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0) sched_finish(sched);
}

int num_sms() {
  static int n[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!n[dev] && cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    n[dev] = 148;
  return n[dev];
}

namespace {
template <int HD>
int attn_fwd_tc_t(const gpt_config& c, const void* q, const void* k, const void* v, void* o,
                  float* lse, int32_t* status, cudaStream_t st) {
  const uint64_t rows = uint64_t(c.batch) * c.n_head * c.seq_len;
  const uint64_t kv_rows = uint64_t(c.batch) * c.n_kv_head * c.seq_len;
  CUtensorMap mq, mk, mv;
  if (!tile_map(&mq, q, rows, HD, HD, 128) || !tile_map(&mk, k, kv_rows, HD, HD, 128) ||
      !tile_map(&mv, v, kv_rows, HD, HD, 128))
    return 1;
  auto kern = attn_fwd_tc_kernel<HD>;
  const int smem = int(FwdSmem<HD>::BYTES);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 1;
  const int n_rows = c.batch * c.n_head;
  const int n_items = ((c.seq_len + 127) / 128 + 1) / 2 * n_rows;
  kern<<<std::min(n_items, num_sms()), kFwdThreads, smem, st>>>(
      mq, mk, mv, static_cast<__nv_bfloat16*>(o), lse, c.n_head, c.n_kv_head, c.seq_len,
      window_span(c), kLog2e / sqrtf(float(HD)), n_rows, status);
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
// The dQ kernel forms D_i (its dO tile is in shared memory) and writes it for
// the dK/dV kernel, which runs after it on the same stream.  Each kernel owns
// its outputs, so no sum needs atomics (deterministic).  The
// gradients of q and k then go back through the per-head RMSNorm,
// dx = r (g - y mean(g y)), and the transposed RoPE rotation, and land in the
// [q | k | v] gradient rows [B*T, 3*H*hd].
// ===========================================================================
namespace {

// slots of the dK/dV kernel's Q and dO rings (a Q tile is read by S^T_j and,
// after the threads have formed dS^T_j, by dK_j)
constexpr int kDkvRingQ = 3, kDkvRingDO = 2;
// slots of the dQ kernel's K and V rings: a K tile is read by S_j early in its
// step and by the dQ product at the end of it, so it stays resident about two
// steps and needs a third slot to be prefetched in time; V only feeds dP_j
constexpr int kDqRingK = 3, kDqRingV = 2;

// One row's gradient w.r.t. its normalised, rotated q or k (TMEM, fp32, HD
// columns at `taddr`, times `scale`) back through RMSNorm (y: the normalised
// row, rr: its 1/rms) and RoPE, written as bf16 into row r of the shared-memory
// tile `out_tile` (for a TMA store).  y, cos and sin come from shared-memory
// tiles of the CTA's 128 rows.  All tiles are stored as TMA writes and reads
// them, with the 128-byte swizzle: y and out [128 x HD] bf16 in 64-column
// chunks, cos / sin [128 x HD/2] fp32 in 32-column chunks (16 KB per chunk).  The row's two
// compute threads split the rotation pairs: thread `half` takes pairs i in
// [half*HD/4, (half+1)*HD/4) and their partners i + HD/2; the mean(g y) of the
// norm is summed across both through `red` (one compute_bar, reached on every
// path).
__device__ __forceinline__ uint32_t tile_unit(int r, int unit) {  // 16-byte unit of row r
  return uint32_t(unit >> 3) * (128 * 128) + r * 128 + (((unit & 7) ^ (r & 7)) << 4);
}
// The RoPE table rows pos0 .. pos0 + 127 ([T, HD/2] fp32 each) as two tiles of
// 128 * HD * 2 bytes (the size of a bf16 [128 x HD] ring slot), loaded onto `bar`
template <int HD>
__device__ __forceinline__ void load_rope_tiles(uint8_t* cos_dst, uint8_t* sin_dst, const CUtensorMap* map_cos,
                                                const CUtensorMap* map_sin, uint64_t* bar, int pos0) {
  tc::mbar_arrive_expect_tx(bar, 2u * 128 * HD * 2);
#pragma unroll
  for (int c = 0; c < HD / 64; ++c) {
    tc::tma_load_2d(cos_dst + c * (128 * 128), map_cos, bar, c * 32, pos0);
    tc::tma_load_2d(sin_dst + c * (128 * 128), map_sin, bar, c * 32, pos0);
  }
}
// One head's share of the row sum sum_c dqkv_c * qkv_c that the backward of
// the norm in front of the QKV projection needs (qkv = the projection's raw
// output).  RoPE is a rotation, so the share of q (or k) is g . x with x the
// rotated raw head and g the gradient reaching it; without QK-norm x is the
// stored head y and the share is g . y = gy.  With QK-norm (y = x r,
// r = 1 / sqrt(mean(x^2) + eps)), g = r (dy - y mean(dy y)) gives
// g . x = sum(dy y) (1 - mean(y^2)) = gy eps r^2: the norm's gradient is
// almost orthogonal to its input.
__device__ __forceinline__ float norm_row_part(float gy, float rr, int qk_norm, float eps) {
  return qk_norm ? gy * eps * rr * rr : gy;
}

template <int HD>
__device__ __forceinline__ float norm_rope_bwd_half(uint32_t taddr, int half, int r, float scale,
                                                   const uint8_t* y_tile, float rr, int qk_norm,
                                                   const uint8_t* cos_tile, const uint8_t* sin_tile,
                                                   uint8_t* out_tile, bool ok, bool write, float* red) {
  constexpr int HALF = HD / 2, Q4 = HD / 4;
  const int i0 = half * Q4;
  float ga[Q4], gb[Q4];
  uint32_t wa[Q4 / 2], wb[Q4 / 2];  // y, kept as packed bf16 pairs
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
      for (int c = 0; c < Q4 / 2; c += 4) {  // 8 bf16 per 16-byte unit
        const uint4 ua = *reinterpret_cast<const uint4*>(y_tile + tile_unit(r, (i0 + 2 * c) / 8));
        const uint4 ub = *reinterpret_cast<const uint4*>(y_tile + tile_unit(r, (HALF + i0 + 2 * c) / 8));
        wa[c] = ua.x; wa[c + 1] = ua.y; wa[c + 2] = ua.z; wa[c + 3] = ua.w;
        wb[c] = ub.x; wb[c + 1] = ub.y; wb[c + 2] = ub.z; wb[c + 3] = ub.w;
      }
#pragma unroll
      for (int i = 0; i < Q4 / 2; ++i) {
        const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wa[i]));
        const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wb[i]));
        part += ga[2 * i] * fa.x + ga[2 * i + 1] * fa.y + gb[2 * i] * fb.x + gb[2 * i + 1] * fb.y;
      }
    }
  }
  red[half * 128 + r] = part;
  compute_bar();
  const float sum_gy = red[r] + red[128 + r];
  const float mean_gy = sum_gy / float(HD);
  if (!ok || !write) return sum_gy;
  uint32_t pa[Q4 / 2], pb[Q4 / 2];
#pragma unroll
  for (int i = 0; i < Q4; i += 4) {  // 4 fp32 per 16-byte unit
    const float4 c4 = *reinterpret_cast<const float4*>(cos_tile + tile_unit(r, (i0 + i) / 4));
    const float4 s4 = *reinterpret_cast<const float4*>(sin_tile + tile_unit(r, (i0 + i) / 4));
    const float cc[4] = {c4.x, c4.y, c4.z, c4.w}, ss[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      float a0 = ga[i + e], a1 = ga[i + e + 1], b0 = gb[i + e], b1 = gb[i + e + 1];
      if (qk_norm) {
        const float2 ya = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wa[(i + e) / 2]));
        const float2 yb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wb[(i + e) / 2]));
        a0 = rr * (a0 - ya.x * mean_gy); a1 = rr * (a1 - ya.y * mean_gy);
        b0 = rr * (b0 - yb.x * mean_gy); b1 = rr * (b1 - yb.y * mean_gy);
      }
      pa[(i + e) / 2] = pack2(a0 * cc[e] + b0 * ss[e], a1 * cc[e + 1] + b1 * ss[e + 1]);
      pb[(i + e) / 2] = pack2(-a0 * ss[e] + b0 * cc[e], -a1 * ss[e + 1] + b1 * cc[e + 1]);
    }
  }
#pragma unroll
  for (int i = 0; i < Q4 / 2; i += 4) {  // 8 bf16 per 16-byte unit
    *reinterpret_cast<uint4*>(out_tile + tile_unit(r, (i0 + 2 * i) / 8)) =
        make_uint4(pa[i], pa[i + 1], pa[i + 2], pa[i + 3]);
    *reinterpret_cast<uint4*>(out_tile + tile_unit(r, (HALF + i0 + 2 * i) / 8)) =
        make_uint4(pb[i], pb[i + 1], pb[i + 2], pb[i + 3]);
  }
  return sum_gy;
}

// After every compute thread has written its rows of the output tiles: fence,
// barrier, and one thread stores `n` tiles of [128 x HD] with TMA at columns
// col[t] of positions pos0 .. pos0 + 127 of sequence b (clipped at T).
template <int HD>
__device__ __forceinline__ void store_tiles(const CUtensorMap* map, uint8_t* const* tiles, const int* col, int n,
                                            int pos0, int b, bool ok) {
  tc::fence_proxy_async_smem();
  compute_bar();
  if (ok && threadIdx.x == 64) {
    for (int t = 0; t < n; ++t)
#pragma unroll
      for (int c = 0; c < HD / 64; ++c) tc::tma_store_3d(map, tiles[t] + c * (128 * 128), col[t] + c * 64, pos0, b);
    tc::bulk_commit();
    tc::bulk_wait_read();  // the tiles' shared memory is released when the CTA ends
  }
}


}  // namespace

namespace {
// dS = P (dP - D) for 32 keys k0 .. k0 + 31 of one query row, with P =
// 2^(s * scale_log2 - lse2) from the S columns `us` and dP from `up`, as 16
// packed bf16 pairs.  MASK: P = 0 outside the row's visible keys [k_lo, k_hi).
template <bool MASK>
__device__ __forceinline__ void ds_row32(const uint32_t (&us)[32], const uint32_t (&up)[32], uint32_t* pk,
                                         uint64_t sc2, uint64_t nl2, uint64_t nd2, int k0, int k_lo, int k_hi) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int i = 2 * e;
    const float2 x = unf2(fma2(f2(__uint_as_float(us[i]), __uint_as_float(us[i + 1])), sc2, nl2));
    float p0 = ex2(x.x), p1 = ex2(x.y);
    if (MASK) {
      if (k0 + i < k_lo || k0 + i >= k_hi) p0 = 0.f;
      if (k0 + i + 1 < k_lo || k0 + i + 1 >= k_hi) p1 = 0.f;
    }
    const float2 r =
        unf2(mul2(f2(p0, p1), add2(f2(__uint_as_float(up[i]), __uint_as_float(up[i + 1])), nd2)));
    pk[e] = pack2(r.x, r.y);
  }
}
// P^T for 32 queries q0 .. q0 + 31 of one key row: p = 2^(s * scale_log2 -
// lse2_q) from the S^T columns `us` and the staged -lse2 (`nl2s`), kept in fp32
// and as 16 packed bf16 pairs.  MASK: P = 0 outside the key's visible queries
// [q_lo, q_hi).
template <bool MASK>
__device__ __forceinline__ void p_col32(const uint32_t (&us)[32], const float* nl2s, float* p, uint32_t (&pk)[16],
                                        float scale_log2, int q0, int q_lo, int q_hi) {
#pragma unroll
  for (int g = 0; g < 8; ++g) {  // 4 queries per group
    const float4 l4 = *reinterpret_cast<const float4*>(nl2s + 4 * g);
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      const int i = 4 * g + e;
      const float2 x = unf2(fma2(f2(__uint_as_float(us[i]), __uint_as_float(us[i + 1])),
                                 f2(scale_log2, scale_log2), e ? f2(l4.z, l4.w) : f2(l4.x, l4.y)));
      float p0 = ex2(x.x), p1 = ex2(x.y);
      if (MASK) {
        if (q0 + i < q_lo || q0 + i >= q_hi) p0 = 0.f;
        if (q0 + i + 1 < q_lo || q0 + i + 1 >= q_hi) p1 = 0.f;
      }
      p[i] = p0;
      p[i + 1] = p1;
      pk[i / 2] = pack2(p0, p1);
    }
  }
}

template <int HD>
struct DqSmem {
  static constexpr uint32_t TILE = 128 * HD * 2;  // a 128-row Q, dO, K or V tile
  static constexpr uint32_t Q_OFF = 0, DO_OFF = TILE;
  static constexpr uint32_t K_OFF = 2 * TILE;                   // K ring
  static constexpr uint32_t V_OFF = K_OFF + kDqRingK * TILE;    // V ring
  static constexpr uint32_t Y_OFF = Q_OFF;   // the Q tile is the y of the norm backward
  // epilogue only, once no product reads K: the norm reduction and the dQ tile
  static constexpr uint32_t RED_OFF = K_OFF, OUT_OFF = K_OFF + TILE;
  // the RoPE tiles of the epilogue, loaded into the V ring once the last dP is done
  static constexpr uint32_t COS_OFF = V_OFF, SIN_OFF = V_OFF + TILE;
  static constexpr uint32_t BAR_OFF = V_OFF + kDqRingV * TILE;
  static constexpr uint32_t DRED_OFF = BAR_OFF + 256;  // the halves of D: 2 x 128 floats
  static constexpr uint32_t BYTES = DRED_OFF + 1024 + 1024;
  static_assert(TILE % 1024 == 0 && BYTES <= 232448, "");
};
struct DqBars {
  uint64_t fixed_full;
  uint64_t k_full[kDqRingK], k_empty[kDqRingK], v_full[kDqRingV], v_empty[kDqRingV];
  uint64_t s_full[2], ds_ready[2];
  uint64_t dp_full, dp_free;
  uint64_t acc_full, epi_full, done, done2;
  uint32_t tmem_base;
  int abort;
};
}  // namespace

// dQ for 128 queries of one (batch, head), looping over 128-key tiles (all
// products M = 128, N = 128: a single issuing warp keeps up with each).  Warp
// 1 issues S_j = Q K_j^T into one of two TMEM S buffers, then dQ += dS_{j-1}
// K_{j-1}; warp 10 issues dP_j = dO V_j^T into the one dP buffer as soon as
// the compute threads have loaded dP_{j-1}.  So S_{j+1} and dP_{j+1} run on
// the tensor core while the threads turn step j into dS.  Compute thread
// (row, half) handles keys [64*half, 64*half + 64) of each tile, in two
// 32-key chunks, and writes bf16 dS into the first 32 of its own 64 S columns:
// the TMEM A operand of the dQ product (its 16-key step k starts at column
// 64*(k/4) + 8*(k%4)), which warp 1 issues before it next overwrites them.
// TMEM: S at columns 0 and 128, dP at 256, dQ at 384.  K and V have separate
// rings (a K tile is also the dQ product's B operand, so it has three slots);
// the Q tile in shared memory doubles as the y of the norm backward, and the
// RoPE tables of its 128 positions are loaded into the V ring after the last dP.
template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_dq_tc_kernel(const __grid_constant__ CUtensorMap map_q128,
                      const __grid_constant__ CUtensorMap map_do128,
                      const __grid_constant__ CUtensorMap map_k128,
                      const __grid_constant__ CUtensorMap map_v128,
                      const __grid_constant__ CUtensorMap map_cos,
                      const __grid_constant__ CUtensorMap map_sin,
                      const __grid_constant__ CUtensorMap map_out,
                      const __nv_bfloat16* __restrict__ o, const float* __restrict__ lse,
                      float* __restrict__ D, const float* __restrict__ rq, int H, int Hkv, int T,
                      int W, float scale, float scale_log2, int qk_norm, float eps,
                      float* __restrict__ npart, int np_stride, int32_t* status) {
  using S = DqSmem<HD>;
  constexpr int NCH = HD / 64;
  constexpr uint32_t CH = 128 * 128;  // bytes of one 64-column chunk of a 128-row tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  DqBars* bars = reinterpret_cast<DqBars*>(smem + S::BAR_OFF);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int n_qt = (T + 127) / 128;
  int bh, rank;
  grouped_item(int(blockIdx.x), int(gridDim.x) / n_qt, n_qt, bh, rank);  // longest first
  const int qt = n_qt - 1 - rank;
  const int b = bh / H, h = bh % H;
  const int q0 = qt * 128;
  const int s_lo = max(0, q0 - W + 1) / 128;  // first key tile with a visible key
  const int n_steps = qt - s_lo + 1;
  const int kv_row_base = (b * Hkv + h / (H / Hkv)) * T;

  ATTN_PROLOGUE(bars, {
    tc::mbar_init(&bars->fixed_full, 1);
    for (int s = 0; s < kDqRingK; ++s) {
      tc::mbar_init(&bars->k_full[s], 1);
      tc::mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kDqRingV; ++s) {
      tc::mbar_init(&bars->v_full[s], 1);
      tc::mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->ds_ready[s], 256);
    }
    tc::mbar_init(&bars->dp_full, 1);
    tc::mbar_init(&bars->dp_free, 256);
    tc::mbar_init(&bars->acc_full, 1);
    tc::mbar_init(&bars->epi_full, 1);
    tc::mbar_init(&bars->done, 1);
    tc::mbar_init(&bars->done2, 1);
  })
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  const uint32_t t_dp = tmem + 256, t_dq = tmem + 384;

  if (warp == 0) {
    // lane 0: Q, dO, then the K ring; lane 1: the V ring
    if (lane < 2) {
      const bool is_k = lane == 0;
      uint64_t* full = is_k ? bars->k_full : bars->v_full;
      uint64_t* empty = is_k ? bars->k_empty : bars->v_empty;
      const CUtensorMap* map = is_k ? &map_k128 : &map_v128;
      uint8_t* base = smem + (is_k ? S::K_OFF : S::V_OFF);
      const int ring = is_k ? kDqRingK : kDqRingV;
      uint32_t issued = 0, last_par = 0;
      if (is_k) {
        tc::mbar_arrive_expect_tx(&bars->fixed_full, 2 * S::TILE);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          tc::tma_load_2d(smem + S::Q_OFF + c * CH, &map_q128, &bars->fixed_full, c * 64, bh * T + q0);
          tc::tma_load_2d(smem + S::DO_OFF + c * CH, &map_do128, &bars->fixed_full, h * HD + c * 64,
                          b * T + q0);
        }
      }
      for (int j = 0; j < n_steps; ++j) {
        const int st = j % ring;
        const uint32_t ph = (j / ring) & 1;
        if (!tc::mbar_wait_bounded(&empty[st], ph ^ 1, abort, kWaitNs)) {
          record_status(status, GPT_ETIMEOUT, K_ATTN, 20);
          *abort = 1;
          break;
        }
        tc::mbar_arrive_expect_tx(&full[st], S::TILE);
#pragma unroll
        for (int c = 0; c < NCH; ++c)
          tc::tma_load_2d(base + st * S::TILE + c * CH, map, &full[st], c * 64,
                          kv_row_base + (s_lo + j) * 128);
        issued |= 1u << st;
        last_par = (last_par & ~(1u << st)) | (ph << st);
      }
      // the V ring is free once every dP is done: the epilogue's RoPE tiles go there
      bool epi = false;
      if (!is_k && !*abort) {
        bool freed = true;
        for (int s = 0; s < ring; ++s)
          if (issued >> s & 1) freed = freed && tc::mbar_wait_bounded(&empty[s], (last_par >> s) & 1, abort, kWaitNs);
        if (freed) {
          load_rope_tiles<HD>(smem + S::COS_OFF, smem + S::SIN_OFF, &map_cos, &map_sin, &bars->epi_full, q0);
          epi = true;
        } else {
          record_status(status, GPT_ETIMEOUT, K_ATTN, 24);
          *abort = 1;
        }
      }
      if (*abort) {
        if (is_k) tc::mbar_wait_bounded(&bars->fixed_full, 0, nullptr, kWaitNs);
        if (epi) tc::mbar_wait_bounded(&bars->epi_full, 0, nullptr, kWaitNs);
        for (int s = 0; s < ring; ++s)
          if (issued >> s & 1) tc::mbar_wait_bounded(&full[s], (last_par >> s) & 1, nullptr, kWaitNs);
      }
    }
  } else if (warp == 1) {
    // S_j = Q K_j^T, then dQ += dS_{j-1} K_{j-1}.  S_j overwrites the dS_{j-2}
    // that this warp's own dQ product read (issued earlier: in order).
    constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t idesc_dq = tc::idesc_bf16_f32(128, HD, false, true);
    const uint64_t qd = tc::smem_desc_sw128(tc::smem_u32(smem + S::Q_OFF), 16);
    bool ok = tc::mbar_spin_warp(&bars->fixed_full, 0, abort, kWaitNs);
    bool issued_any = false;
    auto issue_dq = [&](int j) -> bool {
      if (!tc::mbar_spin_warp(&bars->ds_ready[j & 1], (j >> 1) & 1, abort, kWaitNs)) return false;
      tc::tc_fence_after();
      const uint32_t ds_t = tmem + (j & 1) * 128;
      const uint64_t kb = tc::smem_desc_sw128(tc::smem_u32(smem + S::K_OFF + (j % kDqRingK) * S::TILE), CH);
#pragma unroll
      for (int k = 0; k < 128 / 16; ++k)
        tc::mma_bf16_ts_elect(t_dq, ds_t + 64 * (k >> 2) + 8 * (k & 3), tc::desc_advance(kb, k * 2048),
                              idesc_dq, (j | k) != 0);
      tc::mma_commit_elect(&bars->k_empty[j % kDqRingK]);
      return true;
    };
    for (int j = 0; ok && j < n_steps; ++j) {
      const int st = j % kDqRingK;
      if (!tc::mbar_spin_warp(&bars->k_full[st], (j / kDqRingK) & 1, abort, kWaitNs)) { ok = false; break; }
      tc::tc_fence_after();
      const uint64_t kd = tc::smem_desc_sw128(tc::smem_u32(smem + S::K_OFF + st * S::TILE), 16);
#pragma unroll
      for (int k = 0; k < HD / 16; ++k) {
        const uint32_t off = (k >> 2) * CH + (k & 3) * 32;
        tc::mma_bf16_ss_elect(tmem + (j & 1) * 128, tc::desc_advance(qd, off), tc::desc_advance(kd, off),
                              idesc_s, k != 0);
      }
      issued_any = true;
      tc::mma_commit_elect(&bars->s_full[j & 1]);
      if (j >= 1 && !issue_dq(j - 1)) { ok = false; break; }
    }
    if (ok && n_steps >= 1) ok = issue_dq(n_steps - 1);
    if (ok) tc::mma_commit_elect(&bars->acc_full);
    if (!ok) {
      if (lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 21);
      *abort = 1;
    }
    if (issued_any) {
      tc::mma_commit_elect(&bars->done);
      tc::mbar_wait_warp(&bars->done, 0, nullptr, kWaitNs);
    }
  } else if (warp == 10) {
    // dP_j = dO V_j^T into the dP buffer, once the compute threads have loaded dP_{j-1}
    constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, 128, false, false);
    const uint64_t dod = tc::smem_desc_sw128(tc::smem_u32(smem + S::DO_OFF), 16);
    bool ok = tc::mbar_spin_warp(&bars->fixed_full, 0, abort, kWaitNs);
    bool issued_any = false;
    for (int j = 0; ok && j < n_steps; ++j) {
      const int st = j % kDqRingV;
      if (j >= 1 && !tc::mbar_spin_warp(&bars->dp_free, (j - 1) & 1, abort, kWaitNs)) { ok = false; break; }
      if (!tc::mbar_spin_warp(&bars->v_full[st], (j / kDqRingV) & 1, abort, kWaitNs)) { ok = false; break; }
      tc::tc_fence_after();
      const uint64_t vd = tc::smem_desc_sw128(tc::smem_u32(smem + S::V_OFF + st * S::TILE), 16);
#pragma unroll
      for (int k = 0; k < HD / 16; ++k) {
        const uint32_t off = (k >> 2) * CH + (k & 3) * 32;
        tc::mma_bf16_ss_elect(t_dp, tc::desc_advance(dod, off), tc::desc_advance(vd, off), idesc_s, k != 0);
      }
      issued_any = true;
      tc::mma_commit_elect(&bars->dp_full);
      tc::mma_commit_elect(&bars->v_empty[st]);
    }
    if (!ok) {
      if (lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 23);
      *abort = 1;
    }
    if (issued_any) {
      tc::mma_commit_elect(&bars->done2);
      tc::mbar_wait_warp(&bars->done2, 0, nullptr, kWaitNs);
    }
  } else {
    const Roles R = roles();
    const int q = q0 + R.r;
    const bool qv = q < T;
    // the query's visible keys [k_lo, k_hi): none for a row past T
    const int k_lo = q - W + 1, k_hi = qv ? q + 1 : k_lo;
    const float lse2 = qv ? lse[int64_t(bh) * T + q] * kLog2e : 0.f;
    // D = rowsum(dO o) of this query: each half of the row's columns from the
    // dO tile in shared memory and o in global memory (loaded while the tile
    // is on its way), the halves added in shared memory; written out for the
    // dK/dV kernel
    uint4 ov[HD / 16];
    if (qv) {
      const uint4* orow = reinterpret_cast<const uint4*>(o + (int64_t(b) * T + q) * (int64_t(H) * HD) + h * HD +
                                                         R.half * (HD / 2));
#pragma unroll
      for (int u = 0; u < HD / 16; ++u) ov[u] = __ldg(orow + u);
    }
    bool ok = __all_sync(0xffffffffu, tc::mbar_wait_spin(&bars->fixed_full, 0, abort, kWaitNs));
    float dpart = 0.f;
    if (ok && qv) {
#pragma unroll
      for (int u = 0; u < HD / 16; ++u) {
        const uint4 a = *reinterpret_cast<const uint4*>(smem + S::DO_OFF + tile_unit(R.r, R.half * (HD / 16) + u));
        const uint4 c = ov[u];
        const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wa[e]));
          const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wc[e]));
          dpart = fmaf(x.x, y.x, fmaf(x.y, y.y, dpart));
        }
      }
    }
    float* dred = reinterpret_cast<float*>(smem + S::DRED_OFF);
    dred[R.half * 128 + R.r] = dpart;
    compute_bar();
    const float Dq = dred[R.r] + dred[128 + R.r];
    if (ok && qv && R.half == 0) D[int64_t(bh) * T + q] = Dq;
    if (!ok && R.lane == 0) {
      record_status(status, GPT_ETIMEOUT, K_ATTN, 25);
      *abort = 1;
    }
    for (int j = 0; j < n_steps; ++j) {
      const int sb = j & 1;
      if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_spin(&bars->s_full[sb], (j >> 1) & 1, abort, kWaitNs));
      if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_spin(&bars->dp_full, j & 1, abort, kWaitNs));
      // dP first, so that dP_{j+1} may start as early as possible; S in two
      // 32-column chunks (fewer live registers)
      uint32_t up0[32], up1[32], us[32], pk[32];
      const uint32_t ts = tmem + sb * 128 + R.lane_off + R.half * 64;
      const uint32_t tp = t_dp + R.lane_off + R.half * 64;
      if (ok) {
        tc::tc_fence_after();
        tc::tmem_ld_32x32b_x32(tp, up0);
        tc::tmem_ld_32x32b_x32(tp + 32, up1);
        tc::tmem_ld_32x32b_x32(ts, us);
        tc::tmem_wait_ld();
        tc::tc_fence_before();
      }
      tc::mbar_arrive(&bars->dp_free);  // dP_{j+1} may overwrite the dP columns
      if (ok) {
        const int kb = (s_lo + j) * 128 + R.half * 64;
        const bool need_mask = kb < k_lo || kb + 64 > k_hi;
        const uint64_t sc2 = f2(scale_log2, scale_log2), nl2 = f2(-lse2, -lse2), nd2 = f2(-Dq, -Dq);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (c == 1) {
            tc::tmem_ld_32x32b_x32(ts + 32, us);
            tc::tmem_wait_ld();
          }
          if (need_mask)
            ds_row32<true>(us, c ? up1 : up0, pk + 16 * c, sc2, nl2, nd2, kb + 32 * c, k_lo, k_hi);
          else
            ds_row32<false>(us, c ? up1 : up0, pk + 16 * c, sc2, nl2, nd2, kb + 32 * c, k_lo, k_hi);
        }
        tc::tc_fence_before();  // the chunk-1 load precedes the dS store over the same columns
        tc::tmem_st_32x32b_x32(ts, pk);  // dS over the first 32 of this thread's 64 S columns
        tc::tmem_wait_st();
        tc::tc_fence_before();
      }
      tc::mbar_arrive(&bars->ds_ready[sb]);
    }
    if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_spin(&bars->acc_full, 0, abort, kWaitNs));
    if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_spin(&bars->epi_full, 0, abort, kWaitNs));
    if (!ok) {
      if (R.lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 22);
      *abort = 1;
    } else {
      tc::tc_fence_after();
    }
    const float rrq = qv ? rq[int64_t(bh) * T + q] : 0.f;
    const float gy = norm_rope_bwd_half<HD>(t_dq + R.lane_off, R.half, R.r, scale, smem + S::Y_OFF, rrq,
                                            qk_norm, smem + S::COS_OFF, smem + S::SIN_OFF,
                                            smem + S::OUT_OFF, ok, qv,
                                            reinterpret_cast<float*>(smem + S::RED_OFF));
    if (npart && ok && qv && R.half == 0)  // this head's share of the input norm's row sum
      npart[(int64_t(b) * T + q) * np_stride + h] = norm_row_part(gy, rrq, qk_norm, eps);
    uint8_t* const tiles[1] = {smem + S::OUT_OFF};
    const int cols[1] = {h * HD};
    store_tiles<HD>(&map_out, tiles, cols, 1, q0, b, ok);
  }
  ATTN_EPILOGUE(tmem)
}

namespace {
template <int HD>
struct DkvSmem {
  static constexpr uint32_t TILE = 128 * HD * 2;  // a 128-row K, V, Q or dO tile
  static constexpr uint32_t K_OFF = 0, V_OFF = TILE;
  static constexpr uint32_t Q_OFF = 2 * TILE;                    // Q ring
  static constexpr uint32_t DO_OFF = Q_OFF + kDkvRingQ * TILE;   // dO ring
  static constexpr uint32_t STAT_OFF = DO_OFF + kDkvRingDO * TILE;  // -lse2 x 128 | -D x 128
  // the RoPE tiles of the epilogue, loaded into the dO ring once the last dV is done
  static constexpr uint32_t COS_OFF = DO_OFF, SIN_OFF = DO_OFF + TILE;
  static constexpr uint32_t RED_OFF = STAT_OFF;  // epilogue only, after the last step's stats
  // epilogue only, once no product reads the Q ring: the dV and dK tiles
  static constexpr uint32_t DV_OFF = Q_OFF, DK_OFF = Q_OFF + TILE;
  static constexpr uint32_t VRED_OFF = Q_OFF + 2 * TILE;  // epilogue only: 2 x 128 floats
  static_assert(kDkvRingQ >= 3, "the epilogue's dv . v exchange uses the third Q slot");
  static constexpr uint32_t BAR_OFF = STAT_OFF + 2 * 128 * 4;
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;
  static_assert(TILE % 1024 == 0 && BYTES <= 232448, "");
};
struct DkvBars {
  uint64_t fixed_full;
  uint64_t q_full[kDkvRingQ], q_empty[kDkvRingQ], do_full[kDkvRingDO], do_empty[kDkvRingDO];
  uint64_t stat_full, stat_empty;
  uint64_t s_full, dp_full, p_ready[2], ds_ready;  // p_ready[c]: P^T of query chunk c written
  uint64_t acc_full, epi_full, done;
  uint32_t tmem_base;
  int abort;
};
}  // namespace

// dK, dV for 128 keys of one (batch, kv head), looping over 128-query tiles
// of every query head of its group (all products M = 128, N = 128): S^T_j =
// K Q_j^T, dP^T_j = V dO_j^T, dV += P^T_j dO_j, dK += dS^T_j Q_j, all issued by
// warp 1.  Compute thread (key row, half) handles queries [64*half, 64*half +
// 64) of each tile: it writes bf16 P^T over the first 32 of its 64 S^T columns
// and bf16 dS^T over the first 32 of its dP^T columns (the TMEM A operands of
// the dV and dK products; 16-query step k at column 64*(k/4) + 8*(k%4)).
// While the threads turn S^T_j into P^T_j the tensor core runs dK_{j-1} and
// dP^T_j; while they form dS^T_j it runs dV_j and S^T_{j+1}.  Warp 0 loads K
// and V once and runs the Q and dO rings (a Q tile is read by S^T_j and, a
// step later, by dK_j, so its ring has a third slot); warp 10 stages lse and D
// of each step's queries in shared memory, loading the next step's while the
// threads use the current one.  TMEM: S^T at column 0, dP^T at 128, dV at
// 256, dK at 384.  The K tile in shared memory doubles as the y of the norm
// backward; the RoPE tables of its 128 positions are loaded into the dO ring
// after the last dV.
template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_dkv_tc_kernel(const __grid_constant__ CUtensorMap map_k128,
                       const __grid_constant__ CUtensorMap map_v128,
                       const __grid_constant__ CUtensorMap map_q128,
                       const __grid_constant__ CUtensorMap map_do128,
                       const __grid_constant__ CUtensorMap map_cos,
                       const __grid_constant__ CUtensorMap map_sin,
                       const __grid_constant__ CUtensorMap map_out,
                       const float* __restrict__ lse,
                       const float* __restrict__ D, const float* __restrict__ rk, int H, int Hkv, int T,
                       int W, float scale, float scale_log2, int qk_norm, float eps,
                       float* __restrict__ npart, int np_stride, int32_t* status) {
  using S = DkvSmem<HD>;
  constexpr int NCH = HD / 64;
  constexpr uint32_t CH = 128 * 128;  // bytes of one 64-column chunk of a 128-row tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  DkvBars* bars = reinterpret_cast<DkvBars*>(smem + S::BAR_OFF);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int n_kt = (T + 127) / 128;
  int bkv, kt;  // key tile 0 (the most queries) first
  grouped_item(int(blockIdx.x), int(gridDim.x) / n_kt, n_kt, bkv, kt);
  const int b = bkv / Hkv, hk = bkv % Hkv, rep = H / Hkv;
  const int k0 = kt * 128;
  // queries k0 .. min(T, k0 + 127 + W) - 1 see some key of the tile; the steps
  // run over their 128-query tiles once per query head of the group (head
  // hk*rep + j / n_h)
  const int n_h = (min(T, k0 + 127 + W) + 127) / 128 - kt;
  const int n_steps = rep * n_h;

  ATTN_PROLOGUE(bars, {
    tc::mbar_init(&bars->fixed_full, 1);
    for (int s = 0; s < kDkvRingQ; ++s) {
      tc::mbar_init(&bars->q_full[s], 1);
      tc::mbar_init(&bars->q_empty[s], 1);
    }
    for (int s = 0; s < kDkvRingDO; ++s) {
      tc::mbar_init(&bars->do_full[s], 1);
      tc::mbar_init(&bars->do_empty[s], 1);
    }
    tc::mbar_init(&bars->stat_full, 32);
    tc::mbar_init(&bars->stat_empty, 256);
    tc::mbar_init(&bars->s_full, 1);
    tc::mbar_init(&bars->dp_full, 1);
    tc::mbar_init(&bars->p_ready[0], 256);
    tc::mbar_init(&bars->p_ready[1], 256);
    tc::mbar_init(&bars->ds_ready, 256);
    tc::mbar_init(&bars->acc_full, 1);
    tc::mbar_init(&bars->epi_full, 1);
    tc::mbar_init(&bars->done, 1);
  })
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  const uint32_t t_dp = tmem + 128, t_dv = tmem + 256, t_dk = tmem + 384;

  if (warp == 0) {
    // lane 0: K and V, then the Q ring; lane 1: the dO ring
    if (lane < 2) {
      const bool is_q = lane == 0;
      uint64_t* full = is_q ? bars->q_full : bars->do_full;
      uint64_t* empty = is_q ? bars->q_empty : bars->do_empty;
      uint8_t* base = smem + (is_q ? S::Q_OFF : S::DO_OFF);
      const int ring = is_q ? kDkvRingQ : kDkvRingDO;
      uint32_t issued = 0, last_par = 0;
      if (is_q) {
        tc::mbar_arrive_expect_tx(&bars->fixed_full, 2 * S::TILE);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          tc::tma_load_2d(smem + S::K_OFF + c * CH, &map_k128, &bars->fixed_full, c * 64, bkv * T + k0);
          tc::tma_load_2d(smem + S::V_OFF + c * CH, &map_v128, &bars->fixed_full, c * 64, bkv * T + k0);
        }
      }
      for (int j = 0; j < n_steps; ++j) {
        const int st = j % ring;
        const uint32_t ph = (j / ring) & 1;
        const int gi = j / n_h;
        const int qs = (kt + j - gi * n_h) * 128;
        const int h = hk * rep + gi;
        if (!tc::mbar_wait_bounded(&empty[st], ph ^ 1, abort, kWaitNs)) {
          record_status(status, GPT_ETIMEOUT, K_ATTN, 30);
          *abort = 1;
          break;
        }
        tc::mbar_arrive_expect_tx(&full[st], S::TILE);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          if (is_q)
            tc::tma_load_2d(base + st * S::TILE + c * CH, &map_q128, &full[st], c * 64, (b * H + h) * T + qs);
          else
            tc::tma_load_2d(base + st * S::TILE + c * CH, &map_do128, &full[st], h * HD + c * 64, b * T + qs);
        }
        issued |= 1u << st;
        last_par = (last_par & ~(1u << st)) | (ph << st);
      }
      // the dO ring is free once every dV and dP^T is done: the epilogue's RoPE tiles go there
      bool epi = false;
      if (!is_q && !*abort) {
        bool freed = true;
        for (int s = 0; s < ring; ++s)
          if (issued >> s & 1) freed = freed && tc::mbar_wait_bounded(&empty[s], (last_par >> s) & 1, abort, kWaitNs);
        if (freed) {
          load_rope_tiles<HD>(smem + S::COS_OFF, smem + S::SIN_OFF, &map_cos, &map_sin, &bars->epi_full, k0);
          epi = true;
        } else {
          record_status(status, GPT_ETIMEOUT, K_ATTN, 35);
          *abort = 1;
        }
      }
      if (*abort) {
        if (is_q) tc::mbar_wait_bounded(&bars->fixed_full, 0, nullptr, kWaitNs);
        if (epi) tc::mbar_wait_bounded(&bars->epi_full, 0, nullptr, kWaitNs);
        for (int s = 0; s < ring; ++s)
          if (issued >> s & 1) tc::mbar_wait_bounded(&full[s], (last_par >> s) & 1, nullptr, kWaitNs);
      }
    }
  } else if (warp == 10) {
    // -lse2 and -D of step j's queries (4 per lane), loaded before the wait for
    // the threads to be done with step j-1's
    float* stat = reinterpret_cast<float*>(smem + S::STAT_OFF);
    for (int j = 0; j < n_steps; ++j) {
      const int gi = j / n_h;
      const int qs = (kt + j - gi * n_h) * 128;
      const int bh = b * H + hk * rep + gi;
      float l4[4], d4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qq = qs + lane * 4 + e;
        l4[e] = qq < T ? -lse[int64_t(bh) * T + qq] * kLog2e : 0.f;  // staged negated
        d4[e] = qq < T ? -D[int64_t(bh) * T + qq] : 0.f;
      }
      if (!tc::mbar_wait_warp(&bars->stat_empty, (j & 1) ^ 1, abort, kWaitNs)) {
        if (lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 34);
        *abort = 1;
        break;
      }
      *reinterpret_cast<float4*>(stat + lane * 4) = make_float4(l4[0], l4[1], l4[2], l4[3]);
      *reinterpret_cast<float4*>(stat + 128 + lane * 4) = make_float4(d4[0], d4[1], d4[2], d4[3]);
      tc::mbar_arrive(&bars->stat_full);
    }
  } else if (warp == 1) {
    // The products in the order the step needs them: S^T_0 and dP^T_0 first;
    // then per step dV_j (once P^T_j is written), S^T_{j+1} (over P^T_j's
    // columns, so after dV_j), dK_j (once dS^T_j is written) and dP^T_{j+1}
    // (over dS^T_j's columns, so after dK_j).  One issuing thread keeps that
    // order on the tensor core: S^T_{j+1}, which the threads wait for next,
    // never queues behind dK_j.
    constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t idesc_acc = tc::idesc_bf16_f32(128, HD, false, true);
    const uint64_t kd = tc::smem_desc_sw128(tc::smem_u32(smem + S::K_OFF), 16);
    const uint64_t vd = tc::smem_desc_sw128(tc::smem_u32(smem + S::V_OFF), 16);
    // X^T = F Y^T over HD (F: the fixed K or V tile, Y: a ring tile), into `t`
    auto issue_prod = [&](uint32_t t, uint64_t fd, const uint8_t* y) {
      const uint64_t rd = tc::smem_desc_sw128(tc::smem_u32(y), 16);
#pragma unroll
      for (int k = 0; k < HD / 16; ++k) {
        const uint32_t off = (k >> 2) * CH + (k & 3) * 32;
        tc::mma_bf16_ss_elect(t, tc::desc_advance(fd, off), tc::desc_advance(rd, off), idesc_s, k != 0);
      }
    };
    // acc += A^T B over 16-query steps k of the tile's 128 queries (A: bf16
    // pairs over `t`'s columns, B: a ring tile); `kmask` selects the steps
    auto issue_acc = [&](uint32_t acc, uint32_t t, const uint8_t* bt, bool first, uint32_t kmask) {
      const uint64_t bmn = tc::smem_desc_sw128(tc::smem_u32(bt), CH);
#pragma unroll
      for (int k = 0; k < 128 / 16; ++k)
        if (kmask >> k & 1)
          tc::mma_bf16_ts_elect(acc, t + 64 * (k >> 2) + 8 * (k & 3), tc::desc_advance(bmn, k * 2048),
                                idesc_acc, !(first && k == 0));
    };
    // the threads' first 32-query chunk covers steps 0, 1 (half 0) and 4, 5 (half 1)
    constexpr uint32_t kChunk0 = 0x33u, kChunk1 = 0xCCu;
    auto q_tile = [&](int j) { return smem + S::Q_OFF + (j % kDkvRingQ) * S::TILE; };
    auto do_tile = [&](int j) { return smem + S::DO_OFF + (j % kDkvRingDO) * S::TILE; };
    auto q_ready = [&](int j) { return tc::mbar_spin_warp(&bars->q_full[j % kDkvRingQ], (j / kDkvRingQ) & 1, abort, kWaitNs); };
    auto do_ready = [&](int j) { return tc::mbar_spin_warp(&bars->do_full[j % kDkvRingDO], (j / kDkvRingDO) & 1, abort, kWaitNs); };
    bool ok = tc::mbar_spin_warp(&bars->fixed_full, 0, abort, kWaitNs) && q_ready(0);
    bool issued_any = false;
    if (ok) {
      tc::tc_fence_after();
      issue_prod(tmem, kd, q_tile(0));
      tc::mma_commit_elect(&bars->s_full);
      issued_any = true;
      ok = do_ready(0);
    }
    if (ok) {
      tc::tc_fence_after();
      issue_prod(t_dp, vd, do_tile(0));
      tc::mma_commit_elect(&bars->dp_full);
    }
    for (int j = 0; ok && j < n_steps; ++j) {
      // dV += P^T_j dO_j, the first chunk's steps as soon as the threads have
      // written them, while they form the second
      if (!tc::mbar_spin_warp(&bars->p_ready[0], j & 1, abort, kWaitNs)) { ok = false; break; }
      tc::tc_fence_after();
      issue_acc(t_dv, tmem, do_tile(j), j == 0, kChunk0);
      if (!tc::mbar_spin_warp(&bars->p_ready[1], j & 1, abort, kWaitNs)) { ok = false; break; }
      tc::tc_fence_after();
      issue_acc(t_dv, tmem, do_tile(j), false, kChunk1);
      tc::mma_commit_elect(&bars->do_empty[j % kDkvRingDO]);  // dP^T_j and dV_j read dO_j
      if (j + 1 < n_steps) {
        if (!q_ready(j + 1)) { ok = false; break; }
        tc::tc_fence_after();
        issue_prod(tmem, kd, q_tile(j + 1));  // S^T_{j+1}
        tc::mma_commit_elect(&bars->s_full);
      }
      if (!tc::mbar_spin_warp(&bars->ds_ready, j & 1, abort, kWaitNs)) { ok = false; break; }
      tc::tc_fence_after();
      issue_acc(t_dk, t_dp, q_tile(j), j == 0, 0xFFu);     // dK += dS^T_j Q_j
      tc::mma_commit_elect(&bars->q_empty[j % kDkvRingQ]);  // S^T_j and dK_j read Q_j
      if (j + 1 < n_steps) {
        if (!do_ready(j + 1)) { ok = false; break; }
        tc::tc_fence_after();
        issue_prod(t_dp, vd, do_tile(j + 1));  // dP^T_{j+1}
        tc::mma_commit_elect(&bars->dp_full);
      }
    }
    if (ok) tc::mma_commit_elect(&bars->acc_full);
    if (!ok) {
      if (lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 31);
      *abort = 1;
    }
    if (issued_any) {
      tc::mma_commit_elect(&bars->done);
      tc::mbar_wait_warp(&bars->done, 0, nullptr, kWaitNs);
    }
  } else {
    const Roles R = roles();
    const int key = k0 + R.r;
    const bool kv = key < T;
    // the key's visible queries [q_lo, q_hi): none for a row past T
    const int q_lo = key, q_hi = kv ? min(T, key + W) : key;
    const uint32_t ts = tmem + R.lane_off + R.half * 64;
    const uint32_t tp = t_dp + R.lane_off + R.half * 64;
    const float* stat = reinterpret_cast<const float*>(smem + S::STAT_OFF) + R.half * 64;
    bool ok = true;
    for (int j = 0; j < n_steps; ++j) {
      const int qs = (kt + j - (j / n_h) * n_h) * 128 + R.half * 64;
      if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_spin(&bars->stat_full, j & 1, abort, kWaitNs));
      if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_spin(&bars->s_full, j & 1, abort, kWaitNs));
      const bool need_mask = qs < q_lo || qs + 64 > q_hi;
      float p[64];
      if (ok) {
        tc::tc_fence_after();
        uint32_t us0[32], us1[32];
        tc::tmem_ld_32x32b_x32(ts, us0);
        tc::tmem_ld_32x32b_x32(ts + 32, us1);
        tc::tmem_wait_ld();
        // P^T over the first 32 of this thread's S^T columns (all 64 S^T values
        // are in registers), one 32-query chunk at a time, each announced
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
          if (need_mask)
            p_col32<true>(c ? us1 : us0, stat + 32 * c, p + 32 * c, pk, scale_log2, qs + 32 * c, q_lo, q_hi);
          else
            p_col32<false>(c ? us1 : us0, stat + 32 * c, p + 32 * c, pk, scale_log2, qs + 32 * c, q_lo, q_hi);
          tc::tmem_st_32x32b_x16(ts + 16 * c, pk);
          tc::tmem_wait_st();
          tc::tc_fence_before();
          tc::mbar_arrive(&bars->p_ready[c]);
        }
      } else {
        tc::mbar_arrive(&bars->p_ready[0]);
        tc::mbar_arrive(&bars->p_ready[1]);
      }
      if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_spin(&bars->dp_full, j & 1, abort, kWaitNs));
      if (ok) {
        tc::tc_fence_after();
        // dS^T over the first 32 of this thread's dP^T columns: 16 of them per
        // 32 queries, each written after those columns' dP values were loaded
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t up[32], pd[16];
          tc::tmem_ld_32x32b_x32(tp + 32 * c, up);
          tc::tmem_wait_ld();
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const float4 d4 = *reinterpret_cast<const float4*>(stat + 128 + 32 * c + 4 * g);
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
              const int i = 4 * g + e;
              const float2 r = unf2(mul2(f2(p[32 * c + i], p[32 * c + i + 1]),
                                         add2(f2(__uint_as_float(up[i]), __uint_as_float(up[i + 1])),
                                              e ? f2(d4.z, d4.w) : f2(d4.x, d4.y))));
              pd[i / 2] = pack2(r.x, r.y);
            }
          }
          tc::tmem_st_32x32b_x16(tp + 16 * c, pd);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
      }
      tc::mbar_arrive(&bars->stat_empty);  // this step's lse and D are no longer read
      tc::mbar_arrive(&bars->ds_ready);
    }
    if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait_spin(&bars->acc_full, 0, abort, kWaitNs));
    if (!ok) {
      if (R.lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 32);
      *abort = 1;
    } else {
      tc::tc_fence_after();
    }
    const int d = H * HD;
    float vdot = 0.f;  // this half's sum dv . v (the input norm's row sum, when asked for)
    if (ok) {  // dV: this thread's half of the columns, into the dV tile
#pragma unroll
      for (int c = 0; c < HD / 2; c += 32) {
        float v[32];
        tmem_ld<32>(t_dv + R.lane_off + R.half * (HD / 2) + c, v);
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          const int unit = (R.half * (HD / 2) + c + i) / 8;
          *reinterpret_cast<uint4*>(smem + S::DV_OFF + tile_unit(R.r, unit)) =
              make_uint4(pack2(v[i], v[i + 1]), pack2(v[i + 2], v[i + 3]), pack2(v[i + 4], v[i + 5]),
                         pack2(v[i + 6], v[i + 7]));
          if (npart) {
            const uint4 w = *reinterpret_cast<const uint4*>(smem + S::V_OFF + tile_unit(R.r, unit));
            const uint32_t wu[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wu[e]));
              vdot = fmaf(v[i + 2 * e], f.x, fmaf(v[i + 2 * e + 1], f.y, vdot));
            }
          }
        }
      }
    }
    // the two halves' dv . v meet in the Q ring's third slot (free in the
    // epilogue), ordered by the norm backward's barrier below
    float* vred = reinterpret_cast<float*>(smem + S::VRED_OFF);
    vred[R.half * 128 + R.r] = vdot;
    if (ok && !__all_sync(0xffffffffu, tc::mbar_wait_spin(&bars->epi_full, 0, abort, kWaitNs))) {
      if (R.lane == 0) record_status(status, GPT_ETIMEOUT, K_ATTN, 36);
      *abort = 1;
      ok = false;
    }
    // the stats region is free once every step is done (acc_full): it holds red
    const float rrk = kv ? rk[int64_t(bkv) * T + key] : 0.f;
    const float gy = norm_rope_bwd_half<HD>(t_dk + R.lane_off, R.half, R.r, scale, smem + S::K_OFF, rrk,
                                            qk_norm, smem + S::COS_OFF, smem + S::SIN_OFF,
                                            smem + S::DK_OFF, ok, kv,
                                            reinterpret_cast<float*>(smem + S::RED_OFF));
    if (npart && ok && kv && R.half == 0) {  // this k head's and v head's shares
      float* pr = npart + (int64_t(b) * T + key) * np_stride + H;
      pr[hk] = norm_row_part(gy, rrk, qk_norm, eps);
      pr[Hkv + hk] = vred[R.r] + vred[128 + R.r];
    }
    uint8_t* const tiles[2] = {smem + S::DV_OFF, smem + S::DK_OFF};
    const int cols[2] = {d + (Hkv + hk) * HD, d + hk * HD};
    store_tiles<HD>(&map_out, tiles, cols, 2, k0, b, ok);
  }
  ATTN_EPILOGUE(tmem)
}

namespace {
template <int HD>
int attn_bwd_tc_t(const gpt_config& c, const void* q, const void* k, const void* v, const void* o,
                  const void* dO, const float* lse, const float* rq, const float* rk,
                  const float* cos_t, const float* sin_t, float* Dbuf, void* dqkv, float* npart,
                  int32_t* status, cudaStream_t st) {
  const int H = c.n_head, Hkv = c.n_kv_head, T = c.seq_len, B = c.batch, d = H * HD;
  const int np_stride = H + 2 * Hkv;
  const int W = window_span(c);
  const int64_t ldq = qkv_cols(c);
  const uint64_t rows = uint64_t(B) * H * T, kv_rows = uint64_t(B) * Hkv * T, ntok = uint64_t(B) * T;
  CUtensorMap k128, v128, q128, do128, mcos, msin, mout;
  const bool ok = tile_map(&k128, k, kv_rows, HD, HD, 128) && tile_map(&v128, v, kv_rows, HD, HD, 128) &&
                  tile_map(&q128, q, rows, HD, HD, 128) && tile_map(&do128, dO, ntok, d, d, 128) &&
                  tile_map_f32(&mcos, cos_t, T, HD / 2, HD / 2, 128) &&
                  tile_map_f32(&msin, sin_t, T, HD / 2, HD / 2, 128) && seq_map(&mout, dqkv, B, T, ldq);
  if (!ok) return 1;
  const float scale = 1.f / sqrtf(float(HD));
  const float scale_log2 = scale * kLog2e;
  const int nt = (T + 127) / 128;
  auto kq = attn_dq_tc_kernel<HD>;
  const int smem_q = int(DqSmem<HD>::BYTES);
  if (cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q) != cudaSuccess)
    return 1;
  kq<<<nt * B * H, kThreads, smem_q, st>>>(q128, do128, k128, v128, mcos, msin, mout,
                                           static_cast<const __nv_bfloat16*>(o), lse, Dbuf, rq, H,
                                           Hkv, T, W, scale, scale_log2, c.qk_norm, c.norm_eps, npart,
                                           np_stride, status);
  auto kk = attn_dkv_tc_kernel<HD>;
  const int smem_k = int(DkvSmem<HD>::BYTES);
  if (cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_k) != cudaSuccess)
    return 1;
  kk<<<nt * B * Hkv, kThreads, smem_k, st>>>(k128, v128, q128, do128, mcos, msin, mout, lse, Dbuf, rk, H,
                                                Hkv, T, W, scale, scale_log2, c.qk_norm, c.norm_eps, npart,
                                                np_stride, status);
  return last_launch_rc();
}
}  // namespace

int launch_attn_bwd_tc(const gpt_config& c, const void* q, const void* k, const void* v,
                       const void* o, const void* dO, const float* lse, const float* rq,
                       const float* rk, const float* cos_t, const float* sin_t, float* Dbuf,
                       void* dqkv, float* norm_part, int32_t* status, void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  return c.head_dim == 128
             ? attn_bwd_tc_t<128>(c, q, k, v, o, dO, lse, rq, rk, cos_t, sin_t, Dbuf, dqkv, norm_part, status, st)
             : attn_bwd_tc_t<64>(c, q, k, v, o, dO, lse, rq, rk, cos_t, sin_t, Dbuf, dqkv, norm_part, status, st);
}

}  // namespace gpt
