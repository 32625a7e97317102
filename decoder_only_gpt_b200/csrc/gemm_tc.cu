// bf16 GEMM on the sm_100a tensor cores: C[m,n] = sum_k A(m,k) B(n,k), fp32
// accumulation in tensor memory, with the fused epilogues of the step.
//
// Design: clusters of two CTAs (one per SM), persistent over 256 x 256 output
// tiles, K-block 64 (one 128-byte swizzle atom), 6-stage shared-memory ring:
//   warp 0      TMA producer of each CTA: its 128 rows of A and its 128
//               columns of B per stage; both CTAs' loads complete on the
//               first CTA's stage barrier;
//   warp 1      one thread of the first CTA issues tcgen05.mma.cta_group::2
//               (M=256, N=256, K=16) reading both CTAs' shared memory into one
//               of two 256-column fp32 accumulators (each CTA's TMEM holds its
//               128 rows; 512 columns), and tcgen05.commit frees stages in both
//               CTAs / hands the accumulator to both epilogues;
//   warps 2..9  epilogue of each CTA: two warps per TMEM lane quarter, each
//               thread one row and 128 of the tile's 256 columns; tcgen05.ld
//               32 columns at a time, apply the epilogue, store to global.  The
//               operand bytes the epilogue reads (stored activation, fp32
//               residual) are prefetched into L2 one tile ahead.  Double-buffered
//               TMEM lets the epilogue of tile i overlap the MMAs of tile i+1.
// Each CTA loads only half of B, so a pair moves a third less operand data per
// FLOP than two independent 128 x 256 tiles.  Either operand may be K-major
// (forward: X W^T) or MN-major (dgrad reads W as stored, wgrad reads dY and X
// as stored), selected per operand through the TMA box shape, the smem
// descriptor and the instruction descriptor.  Weight-gradient GEMMs with too
// few tiles to fill the GPU split K (fp32 partials, reduced in a fixed order).
// No load is multicast.  Every wait is bounded (GPT_ETIMEOUT in the status word).
#include <cudaTypedefs.h>

#include "epilogue.cuh"
#include "tc_ptx.cuh"

namespace gpt {

namespace {
constexpr int BN = 256, BK = 64;
constexpr int kThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int EC = 128;          // columns of a tile handled by one epilogue thread
static_assert((kThreads - 64) / 128 * EC == 256, "epilogue warps must cover the tile's columns");
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

}  // namespace

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// Ask L2 for the bytes this thread's epilogue will read for one tile row
// (columns col0 .. col0 + EC): the stored activation (ReLU^2'), the fp32 residual
// (residual add) or the gradient being accumulated.  Issued before the thread
// waits for the tile's accumulator, so the reads hit L2 when the tile lands.
__device__ __forceinline__ void epilogue_prefetch(const GemmArgs& g, int row, int col0, int splits) {
  if (row >= g.M || splits > 1) return;
  const int64_t base = int64_t(row) * g.ldo + col0;
  const int cols = min(EC, g.N - col0);
  if (cols <= 0) return;
  if (g.epi == EPI_DRELU2) {
    const char* p = reinterpret_cast<const char*>(static_cast<const __nv_bfloat16*>(g.aux) + base);
    for (int b = 0; b < cols * 2; b += 128) prefetch_l2(p + b);
  } else if (g.epi == EPI_RESID_F32 || g.epi == EPI_NORM_BWD) {
    const char* p = reinterpret_cast<const char*>(static_cast<const float*>(g.out) + base);
    for (int b = 0; b < cols * 4; b += 128) prefetch_l2(p + b);
    if (g.epi == EPI_NORM_BWD) {
      const char* h = reinterpret_cast<const char*>(static_cast<const __nv_bfloat16*>(g.aux) + base);
      for (int b = 0; b < cols * 2; b += 128) prefetch_l2(h + b);
    }
  } else if (g.epi == EPI_STORE && g.beta) {
    const char* p = reinterpret_cast<const char*>(static_cast<const __nv_bfloat16*>(g.out) + base);
    for (int b = 0; b < cols * 2; b += 128) prefetch_l2(p + b);
  }
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(h);
}

// Epilogue of 32 consecutive columns [col0, col0+32) of one row.
__device__ __forceinline__ void epi_chunk(const GemmArgs& g, int row, int col0, float (&v)[32],
                                          float& ce_max, float& ce_sum, float& ce_tgt,
                                          int tgt, float lse_row) {
  const bool full = col0 + 32 <= g.N;
  const int64_t base = int64_t(row) * g.ldo + col0;
  switch (g.epi) {
    case EPI_CE_FWD: {
      const int nv = min(32, g.n_valid - col0);
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < nv) mx = fmaxf(mx, v[j]);
      if (nv > 0) {
        float nm = fmaxf(ce_max, mx);
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nv) s += __expf(v[j] - nm);
        ce_sum = ce_sum * __expf(ce_max - nm) + s;
        ce_max = nm;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j == tgt && j < nv) ce_tgt = v[j];
      }
      return;
    }
    case EPI_RESID_F32: {
      float* o = static_cast<float*>(g.out) + base;
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          float4 x = *reinterpret_cast<float4*>(o + j);
          x.x += v[j]; x.y += v[j + 1]; x.z += v[j + 2]; x.w += v[j + 3];
          *reinterpret_cast<float4*>(o + j) = x;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < g.N) o[j] += v[j];
      }
      return;
    }
    case EPI_STORE_F32: {
      float* o = static_cast<float*>(g.out) + base;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < g.N) o[j] = v[j];
      return;
    }
    default:
      break;
  }
  // bf16 outputs
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(g.out) + base;
  float r[32];
  switch (g.epi) {
    case EPI_STORE:
      if (g.beta) {
        if (full) {
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint4 u = *reinterpret_cast<const uint4*>(o + j);
            float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y), c = unpack_bf16(u.z),
                   d = unpack_bf16(u.w);
            r[j] = v[j] + a.x; r[j + 1] = v[j + 1] + a.y; r[j + 2] = v[j + 2] + b.x;
            r[j + 3] = v[j + 3] + b.y; r[j + 4] = v[j + 4] + c.x; r[j + 5] = v[j + 5] + c.y;
            r[j + 6] = v[j + 6] + d.x; r[j + 7] = v[j + 7] + d.y;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = v[j] + (col0 + j < g.N ? __bfloat162float(o[j]) : 0.f);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = v[j];
      }
      break;
    case EPI_RELU2:
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float t = fmaxf(v[j], 0.f);
        r[j] = t * t;
      }
      break;
    case EPI_DRELU2: {
      const __nv_bfloat16* a = static_cast<const __nv_bfloat16*>(g.aux) + base;
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          uint4 u = *reinterpret_cast<const uint4*>(a + j);
          float2 p0 = unpack_bf16(u.x), p1 = unpack_bf16(u.y), p2 = unpack_bf16(u.z),
                 p3 = unpack_bf16(u.w);
          r[j] = v[j] * 2.f * sqrt_approx(p0.x); r[j + 1] = v[j + 1] * 2.f * sqrt_approx(p0.y);
          r[j + 2] = v[j + 2] * 2.f * sqrt_approx(p1.x); r[j + 3] = v[j + 3] * 2.f * sqrt_approx(p1.y);
          r[j + 4] = v[j + 4] * 2.f * sqrt_approx(p2.x); r[j + 5] = v[j + 5] * 2.f * sqrt_approx(p2.y);
          r[j + 6] = v[j + 6] * 2.f * sqrt_approx(p3.x); r[j + 7] = v[j + 7] * 2.f * sqrt_approx(p3.y);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          r[j] = col0 + j < g.N ? v[j] * 2.f * sqrt_approx(__bfloat162float(a[j])) : 0.f;
      }
      break;
    }
    case EPI_CE_BWD:
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int n = col0 + j;
        float p = __expf(v[j] - lse_row);
        r[j] = n < g.n_valid ? (p - (n == tgt ? 1.f : 0.f)) * g.inv_n : 0.f;
      }
      break;
    default:
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] = v[j];
      break;
  }
  if (full) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      uint4 u;
      u.x = pack_bf16(r[j], r[j + 1]);
      u.y = pack_bf16(r[j + 2], r[j + 3]);
      u.z = pack_bf16(r[j + 4], r[j + 5]);
      u.w = pack_bf16(r[j + 6], r[j + 7]);
      *reinterpret_cast<uint4*>(o + j) = u;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j < g.N) o[j] = __float2bfloat16_rn(r[j]);
  }
}

// Staging tile of one epilogue warp: 32 rows x 32 fp32, its 16-byte units
// XOR-swizzled by row so that both the row-wise writes and the column-wise
// reads are free of bank conflicts; then one fp32 per row (kStageRowSlot).
constexpr uint32_t kStageBytes = 32 * 32 * 4 + 32 * 4;
constexpr int kStageRowSlot = 32 * 32;
__device__ __forceinline__ float4* stage_at(float* tile, int r, int u) {
  return reinterpret_cast<float4*>(tile + r * 32 + ((u ^ (r & 7)) << 2));
}

// EPI_QKV: a thread's 128 tile columns hold whole heads (head_dim 64 or 128
// divides 128).  For each head of this row: v is copied to its head-major row; q and k
// are rotated by RoPE (pairs (i, i + hd/2)), scaled by 1/rms of the rotated row
// (the rotation keeps the norm, so the sum of squares is taken on the raw row)
// and written head-major, with the 1/rms kept for the backward.
template <bool SCALED>
__device__ __forceinline__ void epi_qkv_row(const GemmArgs& g, uint32_t taddr, int row,
                                            int col_base, bool row_ok, float esc, float* tile) {
  // esc: the operands' dequantization factor of this row (8-bit operands only)
  auto val = [&](uint32_t u) { return SCALED ? u2f(u) * esc : u2f(u); };
  const int hd = g.head_dim, half = hd / 2, H = g.n_head, Hkv = g.n_kv_head, T = g.seq_len;
  const int b = row_ok ? row / T : 0, t = row_ok ? row % T : 0;
  for (int seg = 0; seg < EC / hd; ++seg) {
    const int c0 = col_base + seg * hd;
    if (c0 >= g.N) break;  // uniform across the warp
    // column head c0/hd: the n_head q heads, then n_kv_head k heads, then v heads
    const int ch = c0 / hd;
    const int part = ch < H ? 0 : (ch < H + Hkv ? 1 : 2);
    const int h = part == 0 ? ch : (part == 1 ? ch - H : ch - H - Hkv);
    const int nh = part == 0 ? H : Hkv;  // heads of this part's [B, nh, T, hd] output
    const uint32_t tcol = taddr + seg * hd;
    const int64_t dst = ((int64_t(b) * nh + h) * T + t) * hd;
    if (part == 2) {
      __nv_bfloat16* vo = static_cast<__nv_bfloat16*>(g.v_out) + dst;
      for (int c = 0; c < hd; c += 32) {
        uint32_t u[32];
        tc::tmem_ld_32x32b_x32(tcol + c, u);
        tc::tmem_wait_ld();
        if (!row_ok) continue;
#pragma unroll
        for (int i = 0; i < 32; i += 8)
          *reinterpret_cast<uint4*>(vo + c + i) =
              make_uint4(pack_bf16(val(u[i]), val(u[i + 1])), pack_bf16(val(u[i + 2]), val(u[i + 3])),
                         pack_bf16(val(u[i + 4]), val(u[i + 5])), pack_bf16(val(u[i + 6]), val(u[i + 7])));
      }
      continue;
    }
    float ss = 0.f;
    for (int c = 0; c < hd; c += 32) {
      uint32_t u[32];
      tc::tmem_ld_32x32b_x32(tcol + c, u);
      tc::tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) ss = fmaf(val(u[i]), val(u[i]), ss);
    }
    const float r = g.qk_norm ? rsqrtf(ss / float(hd) + g.norm_eps) : 1.f;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(part == 0 ? g.q_out : g.k_out) + dst;
    // pair-major tables: the warp's lanes hold consecutive positions, so each
    // load instruction reads one contiguous 128-byte line
    const float* cr = g.rope_cos + t;
    const float* sr = g.rope_sin + t;
    const int lane = threadIdx.x & 31;
    for (int i0 = 0; i0 < half; i0 += 16) {
      uint32_t ua[16], ub[16];
      tc::tmem_ld_32x32b_x16(tcol + i0, ua);
      tc::tmem_ld_32x32b_x16(tcol + half + i0, ub);
      tc::tmem_wait_ld();
      float cv[16], sv[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        cv[e] = __ldg(cr + int64_t(i0 + e) * T);
        sv[e] = __ldg(sr + int64_t(i0 + e) * T);
      }
      uint32_t pa[8], pb[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float c0v = cv[2 * e], c1v = cv[2 * e + 1];
        const float s0v = sv[2 * e], s1v = sv[2 * e + 1];
        const float a0 = val(ua[2 * e]), a1 = val(ua[2 * e + 1]);
        const float b0 = val(ub[2 * e]), b1 = val(ub[2 * e + 1]);
        pa[e] = pack_bf16((a0 * c0v - b0 * s0v) * r, (a1 * c1v - b1 * s1v) * r);
        pb[e] = pack_bf16((a0 * s0v + b0 * c0v) * r, (a1 * s1v + b1 * c1v) * r);
      }
      // through the warp's staging tile, so that each store instruction
      // writes 8 rows x 64 contiguous bytes (whole 32-byte sectors) instead of
      // 32 rows x 16 bytes: row r's 32 outputs go to units 0..3 of tile row r,
      // then lane (row 8k + lane/4, unit lane%4) stores one unit
      __syncwarp();
      *reinterpret_cast<uint4*>(stage_at(tile, lane, 0)) = make_uint4(pa[0], pa[1], pa[2], pa[3]);
      *reinterpret_cast<uint4*>(stage_at(tile, lane, 1)) = make_uint4(pa[4], pa[5], pa[6], pa[7]);
      *reinterpret_cast<uint4*>(stage_at(tile, lane, 2)) = make_uint4(pb[0], pb[1], pb[2], pb[3]);
      *reinterpret_cast<uint4*>(stage_at(tile, lane, 3)) = make_uint4(pb[4], pb[5], pb[6], pb[7]);
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int rr = 8 * k + (lane >> 2), u = lane & 3;
        const uint64_t orow = __shfl_sync(0xffffffffu, reinterpret_cast<uint64_t>(out), rr);
        const bool rok = __shfl_sync(0xffffffffu, int(row_ok), rr) != 0;
        const uint4 v = *reinterpret_cast<const uint4*>(stage_at(tile, rr, u));
        if (rok)
          *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(orow) + (u < 2 ? i0 : half + i0) +
                                    8 * (u & 1)) = v;
      }
    }
    if (row_ok) {
      const int64_t ri = (int64_t(b) * nh + h) * T + t;
      (part == 0 ? g.rq : g.rk)[ri] = r;
    }
  }
}


// Partial-column fallback (col + 4 > N, or a row pitch that is not a multiple
// of 4): the same element-wise epilogue, one element at a time.  rs: the
// row's r s (EPI_NORM_BWD, whose staged accumulator is already r acc).
// Returns the row partial sum of acc * aux over these columns (EPI_DRELU2),
// else 0.
__device__ __noinline__ float epi4_scalar(const GemmArgs& g, int row, int col, float4 a, int sp,
                                          int splits, int tgt, float lse_row, int64_t obase,
                                          float rs) {
  const int nc = min(4, g.N - col);
  const float v[4] = {a.x, a.y, a.z, a.w};
  float part = 0.f;
  for (int j = 0; j < nc; ++j) {
    const int n = col + j;
    if (splits > 1) {
      g.splitk[(int64_t(sp) * g.M + row) * g.N + n] = v[j];
      continue;
    }
    const int64_t e = obase + int64_t(row) * g.ldo + n;
    if (g.epi == EPI_RESID_F32) { static_cast<float*>(g.out)[e] += v[j]; continue; }
    if (g.epi == EPI_STORE_F32) { static_cast<float*>(g.out)[e] = v[j]; continue; }
    if (g.epi == EPI_NORM_BWD) {
      float* x = static_cast<float*>(g.out);
      const float h = __bfloat162float(static_cast<const __nv_bfloat16*>(g.aux)[e]);
      const float gv = v[j] - h * rs + x[e];
      x[e] = gv;
      static_cast<__nv_bfloat16*>(g.out2)[e] = __float2bfloat16_rn(gv);
      continue;
    }
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(g.out);
    float r = v[j];
    if (g.epi == EPI_STORE && g.beta) r += __bfloat162float(o[e]);
    if (g.epi == EPI_RELU2) { const float t = fmaxf(v[j], 0.f); r = t * t; }
    if (g.epi == EPI_DRELU2) {
      const float in = __bfloat162float(static_cast<const __nv_bfloat16*>(g.aux)[e]);
      part = fmaf(v[j], in, part);
      r = v[j] * 2.f * sqrt_approx(in);
    }
    if (g.epi == EPI_AXPBY)
      r = g.alpha * v[j] + g.beta_aux * __bfloat162float(static_cast<const __nv_bfloat16*>(g.aux)[e]);
    if (g.epi == EPI_CE_BWD) {
      const float pr = __expf(v[j] - lse_row);
      r = n < g.n_valid ? (pr - (n == tgt ? 1.f : 0.f)) * g.inv_n : 0.f;
    }
    o[e] = __float2bfloat16_rn(r);
  }
  return part;
}

// The lane's partials of acc * aux for its rows 4i + rsub (EPI_DRELU2 with
// norm_part_out).
struct NormRows {
  float part[8];
};

// Element-wise epilogue of one 32-column chunk of a warp's 32 rows, from the
// staging tile: lane (rsub, u4) handles columns col .. col + 4 of rows
// 4i + rsub, i = 0..7, so each warp instruction covers 4 rows x 32 columns.
// All of a lane's input loads are issued before any result is stored.
// KIND: an Epilogue value, or -1 for the fp32 partial of a K split.
template <int KIND>
__device__ __forceinline__ void epi_chunk_coalesced(const GemmArgs& g, float* tile, int wrow0, int col,
                                                    int rsub, int u4, int sp, int splits, int tgt,
                                                    float lse_row, int64_t obase, NormRows& nrm) {
  float4 a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = *stage_at(tile, 4 * i + rsub, u4);
  const bool col_ok = col < g.N;
  const bool vec = col + 4 <= g.N && ((KIND == -1 ? g.N : g.ldo) & 3) == 0;
  int t[8];
  float ls[8];
  if (KIND == EPI_CE_BWD) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      t[i] = __shfl_sync(0xffffffffu, tgt, 4 * i + rsub);
      ls[i] = __shfl_sync(0xffffffffu, lse_row, 4 * i + rsub);
    }
  }
  if (!col_ok) return;
  if (!vec) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (wrow0 + 4 * i + rsub < g.M)
        nrm.part[i] += epi4_scalar(g, wrow0 + 4 * i + rsub, col, a[i], sp, splits,
                                   KIND == EPI_CE_BWD ? t[i] : -1, KIND == EPI_CE_BWD ? ls[i] : 0.f,
                                   obase, KIND == EPI_NORM_BWD ? tile[kStageRowSlot + 4 * i + rsub] : 0.f);
    return;
  }
  bool ok[8];
  int64_t e[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = wrow0 + 4 * i + rsub;
    ok[i] = row < g.M;
    e[i] = KIND == -1 ? (int64_t(sp) * g.M + row) * g.N + col : obase + int64_t(row) * g.ldo + col;
  }
  if (KIND == -1 || KIND == EPI_STORE_F32 || KIND == EPI_RESID_F32) {
    float* o = KIND == -1 ? g.splitk : static_cast<float*>(g.out);
    if (KIND == EPI_RESID_F32) {
      float4 x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = ok[i] ? *reinterpret_cast<const float4*>(o + e[i]) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        a[i].x += x[i].x; a[i].y += x[i].y; a[i].z += x[i].z; a[i].w += x[i].w;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (ok[i]) *reinterpret_cast<float4*>(o + e[i]) = a[i];
    return;
  }
  if (KIND == EPI_NORM_BWD) {
    // x <- x + r acc - (r s) h (the staged values are r acc; r s per row in
    // the staging tile's row slots), and its bf16 copy
    float* xo = static_cast<float*>(g.out);
    const __nv_bfloat16* hs = static_cast<const __nv_bfloat16*>(g.aux);
    __nv_bfloat16* o2 = static_cast<__nv_bfloat16*>(g.out2);
    // two halves of 4 rows: every load of a half issued before its stores
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float4 x[4];
      uint2 hw[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = 4 * half + q;
        x[q] = ok[i] ? *reinterpret_cast<const float4*>(xo + e[i]) : make_float4(0.f, 0.f, 0.f, 0.f);
        hw[q] = ok[i] ? *reinterpret_cast<const uint2*>(hs + e[i]) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = 4 * half + q;
        const float rs = tile[kStageRowSlot + 4 * i + rsub];
        const float2 h0 = unpack_bf16(hw[q].x), h1 = unpack_bf16(hw[q].y);
        float4 r;
        r.x = fmaf(-rs, h0.x, a[i].x) + x[q].x;
        r.y = fmaf(-rs, h0.y, a[i].y) + x[q].y;
        r.z = fmaf(-rs, h1.x, a[i].z) + x[q].z;
        r.w = fmaf(-rs, h1.y, a[i].w) + x[q].w;
        if (ok[i]) {
          *reinterpret_cast<float4*>(xo + e[i]) = r;
          *reinterpret_cast<uint2*>(o2 + e[i]) = make_uint2(pack_bf16(r.x, r.y), pack_bf16(r.z, r.w));
        }
      }
    }
    return;
  }
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(g.out);
  constexpr bool kIn = KIND == EPI_DRELU2 || KIND == EPI_STORE || KIND == EPI_AXPBY;
  uint2 w[8];
  if (kIn && (KIND != EPI_STORE || g.beta)) {
    const __nv_bfloat16* src = KIND == EPI_STORE ? o : static_cast<const __nv_bfloat16*>(g.aux);
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = ok[i] ? *reinterpret_cast<const uint2*>(src + e[i]) : make_uint2(0u, 0u);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = make_uint2(0u, 0u);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float v[4] = {a[i].x, a[i].y, a[i].z, a[i].w};
    const float2 i0 = unpack_bf16(w[i].x), i1 = unpack_bf16(w[i].y);
    const float in[4] = {i0.x, i0.y, i1.x, i1.y};
    float r[4];
    if (KIND == EPI_DRELU2 && ok[i])
      nrm.part[i] = fmaf(v[0], in[0], fmaf(v[1], in[1], fmaf(v[2], in[2], fmaf(v[3], in[3], nrm.part[i]))));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (KIND == EPI_STORE) r[j] = v[j] + in[j];
      else if (KIND == EPI_RELU2) { const float tt = fmaxf(v[j], 0.f); r[j] = tt * tt; }
      else if (KIND == EPI_DRELU2) r[j] = v[j] * 2.f * sqrt_approx(in[j]);
      else if (KIND == EPI_AXPBY) r[j] = g.alpha * v[j] + g.beta_aux * in[j];
      else if (KIND == EPI_CE_BWD) {
        const int n = col + j;
        const float pr = __expf(v[j] - ls[i]);
        r[j] = n < g.n_valid ? (pr - (n == t[i] ? 1.f : 0.f)) * g.inv_n : 0.f;
      } else r[j] = v[j];
    }
    if (ok[i]) *reinterpret_cast<uint2*>(o + e[i]) = make_uint2(pack_bf16(r[0], r[1]), pack_bf16(r[2], r[3]));
  }
}

// The element-wise epilogues of one thread's EC columns (KIND: an Epilogue
// value, or -1 for the fp32 partials of a K split).  The warp's 32 rows x 32
// columns pass through its staging tile, then each lane handles 4 columns of
// a row so that a warp instruction covers 4 rows x 32 consecutive columns.
// EPI_NORM_BWD: the thread stages r acc for its row and leaves r s in its
// row slot of the staging tile.  EPI_DRELU2 with norm_part_out: each chunk's
// lane partials reduced over the row's 8 lanes, lane u4 keeping row
// 4 u4 + rsub's running sum.
template <int KIND, bool SCALED>
__device__ __forceinline__ void epi_tile_coalesced(const GemmArgs& g, uint32_t taddr, int row, bool row_ok,
                                                   int wrow0, int col_base, int part, int sp, int splits,
                                                   int lane, float* tile, int64_t obase, float esc) {
  const int rsub = lane >> 3, u4 = lane & 7;
  float r_row = 1.f;
  if (KIND == EPI_NORM_BWD) {
    // s = scale * (the row's partials, summed in order)
    float s_row = 0.f;
    r_row = 0.f;
    if (row_ok) {
      const float* pp = g.norm_part + int64_t(row) * g.n_npart;
#pragma unroll 4
      for (int p = 0; p < g.n_npart; ++p) s_row += pp[p];
      s_row *= g.norm_scale;
      r_row = g.norm_r[row];
    }
    tile[kStageRowSlot + lane] = r_row * s_row;  // read after the first chunk's __syncwarp
  }
  const bool want_part = KIND == EPI_DRELU2 && g.norm_part_out != nullptr;
  float psum = 0.f;
  // EPI_DRELU2: the stored activation of chunk c + 1 is prefetched into L1
  // while chunk c is processed (lane l: row l's 64 bytes of the chunk), so
  // the chunk's loads hit L1 instead of waiting on L2
  const __nv_bfloat16* l1_row =
      KIND == EPI_DRELU2 && row_ok ? static_cast<const __nv_bfloat16*>(g.aux) + obase + int64_t(row) * g.ldo
                                   : nullptr;
  if (l1_row && col_base < g.N) prefetch_l1(l1_row + col_base);
#pragma unroll 1
  for (int c = 0; c < EC / 32; ++c) {
    if (l1_row && c + 1 < EC / 32 && col_base + (c + 1) * 32 < g.N)
      prefetch_l1(l1_row + col_base + (c + 1) * 32);
    uint32_t u[32];
    tc::tmem_ld_32x32b_x32(taddr + c * 32, u);
    tc::tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float4 v4 = make_float4(u2f(u[4 * k]), u2f(u[4 * k + 1]), u2f(u[4 * k + 2]), u2f(u[4 * k + 3]));
      if constexpr (SCALED) { v4.x *= esc; v4.y *= esc; v4.z *= esc; v4.w *= esc; }
      if constexpr (KIND == EPI_NORM_BWD) { v4.x *= r_row; v4.y *= r_row; v4.z *= r_row; v4.w *= r_row; }
      *stage_at(tile, lane, k) = v4;
    }
    __syncwarp();
    NormRows nrm;
#pragma unroll
    for (int i = 0; i < 8; ++i) nrm.part[i] = 0.f;
    epi_chunk_coalesced<KIND>(g, tile, wrow0, col_base + c * 32 + 4 * u4, rsub, u4, sp, splits, -1, 0.f,
                              obase, nrm);
    if (want_part) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float p = nrm.part[i];
        p += __shfl_xor_sync(0xffffffffu, p, 1);
        p += __shfl_xor_sync(0xffffffffu, p, 2);
        p += __shfl_xor_sync(0xffffffffu, p, 4);
        if (u4 == i) psum += p;
      }
    }
    __syncwarp();
  }
  if (want_part && part < g.n_npart) {
    const int r = wrow0 + 4 * u4 + rsub;
    if (r < g.M) g.norm_part_out[int64_t(r) * g.n_npart + part] = psum;
  }
}

// Epilogue of one accumulator tile for one thread: row row0 + 32*quarter +
// lane, columns col_base .. col_base + EC (TMEM columns taddr ..), K split sp
// of `splits`; `part` indexes this column block's cross-entropy partials.
template <bool SCALED>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& g, uint32_t taddr, int row0,
                                              int col_base, int part, int sp, int splits,
                                              int quarter, int lane, float* tile, int64_t obase) {
  const int row = row0 + quarter * 32 + lane;
  const bool row_ok = row < g.M;
  // 8-bit operands: the accumulator times the row's and the weight's
  // dequantization factors (powers of two)
  float esc = 1.f;
  if constexpr (SCALED) esc = (row_ok ? g.a_row_scale[row] : 0.f) * *g.b_scale;
  int tgt = -1;
  float lse_row = 0.f;
  if (row_ok && (g.epi == EPI_CE_FWD || g.epi == EPI_CE_BWD)) {
    tgt = g.targets[row];
    if (g.epi == EPI_CE_BWD) lse_row = g.lse[row];
  }
  float ce_max = -INFINITY, ce_sum = 0.f, ce_tgt = 0.f;
  if (g.epi == EPI_QKV) {
    epi_qkv_row<SCALED>(g, taddr, row, col_base, row_ok, esc, tile);
    return;
  }
  if ((g.epi == EPI_CE_FWD || g.epi == EPI_CE_BWD) && splits == 1) {
    // per-row target and lse (or row reductions): each thread keeps its own row
#pragma unroll 1
    for (int c = 0; c < EC / 32; ++c) {
      uint32_t u[32];
      tc::tmem_ld_32x32b_x32(taddr + c * 32, u);
      tc::tmem_wait_ld();
      const int col0 = col_base + c * 32;
      if (row_ok && col0 < g.N) {
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = u2f(u[j]);
        epi_chunk(g, row, col0, v, ce_max, ce_sum, ce_tgt, tgt, lse_row);
      }
    }
  } else {
    const int wrow0 = row0 + quarter * 32;
    switch (splits > 1 ? -1 : int(g.epi)) {
      case -1: epi_tile_coalesced<-1, SCALED>(g, taddr, row, row_ok, wrow0, col_base, part, sp, splits, lane, tile, obase, esc); break;
      case EPI_RESID_F32: epi_tile_coalesced<EPI_RESID_F32, SCALED>(g, taddr, row, row_ok, wrow0, col_base, part, sp, splits, lane, tile, obase, esc); break;
      case EPI_STORE_F32: epi_tile_coalesced<EPI_STORE_F32, SCALED>(g, taddr, row, row_ok, wrow0, col_base, part, sp, splits, lane, tile, obase, esc); break;
      case EPI_RELU2: epi_tile_coalesced<EPI_RELU2, SCALED>(g, taddr, row, row_ok, wrow0, col_base, part, sp, splits, lane, tile, obase, esc); break;
      case EPI_DRELU2: epi_tile_coalesced<EPI_DRELU2, SCALED>(g, taddr, row, row_ok, wrow0, col_base, part, sp, splits, lane, tile, obase, esc); break;
      case EPI_AXPBY: epi_tile_coalesced<EPI_AXPBY, SCALED>(g, taddr, row, row_ok, wrow0, col_base, part, sp, splits, lane, tile, obase, esc); break;
      case EPI_NORM_BWD: epi_tile_coalesced<EPI_NORM_BWD, SCALED>(g, taddr, row, row_ok, wrow0, col_base, part, sp, splits, lane, tile, obase, esc); break;
      default: epi_tile_coalesced<EPI_STORE, SCALED>(g, taddr, row, row_ok, wrow0, col_base, part, sp, splits, lane, tile, obase, esc); break;
    }
  }
  if (row_ok && g.epi == EPI_CE_FWD) {
    g.part_max[int64_t(row) * g.n_part + part] = ce_max;
    g.part_sum[int64_t(row) * g.n_part + part] = ce_sum;
    if (tgt >= col_base && tgt < col_base + EC && tgt < g.n_valid) g.tgt_logit[row] = ce_tgt;
  }
}

// ---------------------------------------------------------------------------
// CTA-pair variant: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256 across the pair).  Each CTA loads its own
// 128 rows of A and its own 128 columns of B (32 KB per stage, 6 stages); the
// loads of both CTAs complete on the first CTA's stage barrier, whose MMA
// thread then issues the pair MMA reading both CTAs' shared memory.  Each
// CTA's TMEM receives its 128 output rows; the epilogue is the same as above.
// No load is multicast.
// ---------------------------------------------------------------------------
namespace {
constexpr int P_BM = 256, P_STAGES = 6;
constexpr uint32_t P_HALF = 128 * BK * 2;  // one CTA's A or B half of a stage: 16 KB
struct __align__(8) PairTail {
  uint64_t full[P_STAGES];
  uint64_t empty[P_STAGES];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kPairTailBytes = (sizeof(PairTail) + 15) / 16 * 16;
constexpr size_t kPairSmemBytes =
    1024 + P_STAGES * 2 * P_HALF + kPairTailBytes + (kThreads - 64) / 32 * kStageBytes;
static_assert(kPairSmemBytes <= 232448, "");
}  // namespace

template <bool AMN, bool BMN, bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a,
                     const __grid_constant__ CUtensorMap map_b, const __grid_constant__ GemmArgs g,
                     int splits) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* smA = smem;
  uint8_t* smB = smem + P_STAGES * P_HALF;
  PairTail* tail = reinterpret_cast<PairTail*>(smem + 2 * P_STAGES * P_HALF);

  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const int m_tiles = (g.M + P_BM - 1) / P_BM, n_tiles = (g.N + BN - 1) / BN;
  const int mn_tiles = m_tiles * n_tiles;  // per product; `g.batch` products
  const int num_units = mn_tiles * g.batch * splits;
  // a K-block is one 128-byte swizzle row of each operand: 64 bf16 or 128 e4m3
  constexpr int BKE = F8 ? 2 * BK : BK;
  static_assert(!F8 || (!AMN && !BMN), "8-bit operands are K-major");
  const int num_kb = (g.K + BKE - 1) / BKE;
  const int kb_per = (num_kb + splits - 1) / splits;
  constexpr uint32_t idesc =
      F8 ? tc::idesc_e4m3_f32(P_BM, BN, AMN, BMN) : tc::idesc_bf16_f32(P_BM, BN, AMN, BMN);

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      tc::mbar_init(&tail->full[s], 1);
      tc::mbar_init(&tail->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&tail->tmem_full[a], 1);
      tc::mbar_init(&tail->tmem_empty[a], 2 * (kThreads - 64));  // both CTAs' epilogue threads
    }
    tc::mbar_init(&tail->mma_done, 1);
    tail->abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc_pair(&tail->tmem_base, TMEM_COLS);
    tc::tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&map_a);
    tc::tma_prefetch_desc(&map_b);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::cluster_sync();  // the peer's barriers exist before anything arrives on them
  tc::tc_fence_after();
  const uint32_t tmem_base = tail->tmem_base;
  volatile int* abort = &tail->abort;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int unit = pair; unit < num_units && !*abort; unit += num_pairs) {
        const int tile = unit / splits, sp = unit % splits;
        const int bi = tile / mn_tiles, mb = (tile % mn_tiles) / n_tiles, nb = tile % n_tiles;
        const int m0 = mb * P_BM + int(rank) * 128, n0 = nb * BN + int(rank) * 128;
        const int ay = int(bi * g.a_bstride), by = int(bi * g.b_bstride);  // batch row offsets
        const int kb_hi = min(num_kb, (sp + 1) * kb_per);
        for (int kb = sp * kb_per; kb < kb_hi; ++kb) {
          if (!tc::mbar_wait_bounded(&tail->empty[stage], phase ^ 1, abort, kWaitLimitNs)) {
            record_status(g.status, GPT_ETIMEOUT, K_GEMM_TC, 11);
            *abort = 1;
            break;
          }
          if (leader) tc::mbar_arrive_expect_tx(&tail->full[stage], 4 * P_HALF);
          const uint32_t bar = tc::mapa_shared(tc::smem_u32(&tail->full[stage]), 0);
          uint8_t* a_dst = smA + stage * P_HALF;
          uint8_t* b_dst = smB + stage * P_HALF;
          if (AMN) {
            tc::tma_load_2d_pair(a_dst, &map_a, bar, m0, ay + kb * BKE);
            tc::tma_load_2d_pair(a_dst + 8192, &map_a, bar, m0 + 64, ay + kb * BKE);
          } else {
            tc::tma_load_2d_pair(a_dst, &map_a, bar, kb * BKE, ay + m0);
          }
          if (BMN) {
            tc::tma_load_2d_pair(b_dst, &map_b, bar, n0, by + kb * BKE);
            tc::tma_load_2d_pair(b_dst + 8192, &map_b, bar, n0 + 64, by + kb * BKE);
          } else {
            tc::tma_load_2d_pair(b_dst, &map_b, bar, kb * BKE, by + n0);
          }
          if (++stage == P_STAGES) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // the leader's whole warp runs the MMA loop; elect.sync issues
    if (leader) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool issued_any = false, failed = false;
      for (int unit = pair; unit < num_units; unit += num_pairs, ++local) {
        if (__any_sync(0xffffffffu, *abort != 0)) break;
        const int sp = unit % splits;
        const int kb_lo = sp * kb_per, kb_hi = min(num_kb, (sp + 1) * kb_per);
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!tc::mbar_wait_warp(&tail->tmem_empty[acc], acc_phase ^ 1, abort, kWaitLimitNs)) {
          if (lane == 0) record_status(g.status, GPT_ETIMEOUT, K_GEMM_TC, 12);
          failed = true;
          break;
        }
        tc::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
          if (!tc::mbar_wait_warp(&tail->full[stage], phase, abort, kWaitLimitNs)) {
            if (lane == 0) record_status(g.status, GPT_ETIMEOUT, K_GEMM_TC, 13);
            failed = true;
            break;
          }
          tc::tc_fence_after();
          const uint64_t da0 = tc::smem_desc_sw128(tc::smem_u32(smA + stage * P_HALF), AMN ? 8192 : 16);
          const uint64_t db0 = tc::smem_desc_sw128(tc::smem_u32(smB + stage * P_HALF), BMN ? 8192 : 16);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {  // 32 bytes of K per MMA, either type
            if constexpr (F8)
              tc::mma_f8_ss_pair_elect(d_tmem, tc::desc_advance(da0, k * 32), tc::desc_advance(db0, k * 32),
                                       idesc, (kb != kb_lo) || k != 0);
            else
              tc::mma_bf16_ss_pair_elect(d_tmem, tc::desc_advance(da0, AMN ? k * 2048 : k * 32),
                                         tc::desc_advance(db0, BMN ? k * 2048 : k * 32), idesc,
                                         (kb != kb_lo) || k != 0);
          }
          issued_any = true;
          const uint32_t e = tc::smem_u32(&tail->empty[stage]);
          tc::mma_commit_pair_elect(e);
          tc::mma_commit_pair_elect(tc::mapa_shared(e, 1));
          if (++stage == P_STAGES) { stage = 0; phase ^= 1; }
        }
        if (failed) break;
        const uint32_t f = tc::smem_u32(&tail->tmem_full[acc]);
        tc::mma_commit_pair_elect(f);
        tc::mma_commit_pair_elect(tc::mapa_shared(f, 1));
      }
      if (failed && lane == 0) *abort = 1;
      if (issued_any) {
        tc::mma_commit_pair_elect(tc::smem_u32(&tail->mma_done));
        tc::mbar_wait_warp(&tail->mma_done, 0, nullptr, kWaitLimitNs);
      }
    }
  } else {
    const int quarter = warp & 3;      // TMEM lanes 32*quarter .. +31
    const int ch = (warp - 2) >> 2;    // columns ch*EC .. ch*EC + EC of each tile
    float* stage_tile = reinterpret_cast<float*>(smem + 2 * P_STAGES * P_HALF + kPairTailBytes +
                                                 (warp - 2) * kStageBytes);
    const int my_row = int(rank) * 128 + quarter * 32 + lane;  // within a 256-row pair tile
    if (pair < num_units && g.batch == 1)
      epilogue_prefetch(g, (pair / splits / n_tiles) * P_BM + my_row,
                        ((pair / splits) % n_tiles) * BN + ch * EC, splits);
    int local = 0;
    for (int unit = pair; unit < num_units; unit += num_pairs, ++local) {
      const int tile = unit / splits, sp = unit % splits;
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      // one tile ahead: the rows of the next unit
      const int next = unit + num_pairs;
      if (next < num_units && g.batch == 1)
        epilogue_prefetch(g, (next / splits / n_tiles) * P_BM + my_row,
                          ((next / splits) % n_tiles) * BN + ch * EC, splits);
      const bool ok = tc::mbar_wait_bounded(&tail->tmem_full[acc], acc_phase, abort, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) record_status(g.status, GPT_ETIMEOUT, K_GEMM_TC, 14);
        *abort = 1;
        break;
      }
      tc::tc_fence_after();
      const int bi = tile / mn_tiles, nb = tile % n_tiles;
      epilogue_tile<F8>(g, tmem_base + (uint32_t(quarter * 32) << 16) + acc * BN + ch * EC,
                    ((tile % mn_tiles) / n_tiles) * P_BM + int(rank) * 128, nb * BN + ch * EC,
                    nb * (BN / EC) + ch, sp, splits, quarter, lane, stage_tile,
                    int64_t(bi) * g.o_bstride * g.ldo);
      tc::tc_fence_before();
      tc::mbar_arrive_cluster(tc::mapa_shared(tc::smem_u32(&tail->tmem_empty[acc]), 0));
    }
  }

  __syncwarp();
  tc::tc_fence_before();
  __syncthreads();
  tc::cluster_sync();  // neither CTA leaves while the pair MMAs may read its shared memory
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;  // resolved once per process
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D tensor [outer, inner] (inner contiguous, row pitch ld elements) of bf16,
// or of one-byte elements (e4m3 codes) when `bytes1`; box [box_outer,
// box_inner], 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
              uint32_t box_inner, uint32_t box_outer, bool bytes1 = false) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * (bytes1 ? 1 : 2)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, bytes1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool AMN, bool BMN, bool F8 = false>
int launch_pair(const GemmArgs& g, int grid, int splits, cudaStream_t st) {
  CUtensorMap ma, mb;
  // batched products: the maps span every product's rows of the stacked arrays
  const uint64_t a_extra = uint64_t(g.batch - 1) * g.a_bstride, b_extra = uint64_t(g.batch - 1) * g.b_bstride;
  constexpr uint32_t KB = F8 ? 128 : 64;  // K-block in elements: 128 bytes
  bool ok = AMN ? make_map(&ma, g.A, g.M, g.K + a_extra, g.lda, 64, 64)
                : make_map(&ma, g.A, g.K, g.M + a_extra, g.lda, KB, 128, F8);
  ok = ok && (BMN ? make_map(&mb, g.B, g.N, g.K + b_extra, g.ldb, 64, 64)
                  : make_map(&mb, g.B, g.K, g.N + b_extra, g.ldb, KB, 128, F8));
  if (!ok) return 1;
  auto kern = gemm_pair_kernel<AMN, BMN, F8>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kPairSmemBytes)) !=
      cudaSuccess)
    return 1;
  kern<<<grid, kThreads, kPairSmemBytes, st>>>(ma, mb, g, splits);
  return last_launch_rc();
}

// out[i] (+)= sum_s partial[s][i], s in order 0..splits-1, stored as bf16
__global__ void splitk_reduce_kernel(const float* __restrict__ part, __nv_bfloat16* __restrict__ out,
                                     int64_t n4, int splits, int beta) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  float4 a = reinterpret_cast<const float4*>(part)[i];
  for (int s = 1; s < splits; ++s) {
    float4 b = reinterpret_cast<const float4*>(part + int64_t(s) * n4 * 4)[i];
    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
  }
  uint2* o = reinterpret_cast<uint2*>(out) + i;
  if (beta) {
    uint2 prev = *o;
    float2 p0 = unpack_bf16(prev.x), p1 = unpack_bf16(prev.y);
    a.x += p0.x; a.y += p0.y; a.z += p1.x; a.w += p1.y;
  }
  *o = make_uint2(pack_bf16(a.x, a.y), pack_bf16(a.z, a.w));
}

int num_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace

// K splits for a GEMM: only plain stores into a contiguous [M, N] output with a
// split-K buffer, and only when the pair-tile count alone would leave SM pairs
// idle; the smallest split count that fills >= 90 % of the waves, keeping >= 8
// k-blocks per split and the partials within the buffer.
int gemm_tc_splits(const GemmArgs& g) {
  if (g.epi != EPI_STORE || !g.splitk || g.ldo != g.N || (g.N & 3) || g.batch != 1 || g.fp8) return 1;
  const int pairs = num_sms() / 2;
  const int tiles = ((g.M + P_BM - 1) / P_BM) * ((g.N + BN - 1) / BN);
  const int num_kb = (g.K + BK - 1) / BK;
  if (tiles >= 3 * pairs) return 1;
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= 4; ++s) {
    if (num_kb / s < 8 || int64_t(s) * g.M * g.N > g.splitk_floats) break;
    const int units = tiles * s;
    const int waves = (units + pairs - 1) / pairs;
    const double eff = double(units) / (double(waves) * pairs);
    if (eff > best_eff + 1e-9) { best_eff = eff; best = s; }
    if (eff >= 0.9) break;
  }
  if (best > 1) {  // every split non-empty: ceil(num_kb / ceil(num_kb / best)) splits
    const int kb_per = (num_kb + best - 1) / best;
    best = (num_kb + kb_per - 1) / kb_per;
  }
  return best;
}

int launch_gemm_tc(const GemmArgs& g_in, void* stream) {
  GemmArgs g = g_in;
  cudaStream_t st = (cudaStream_t)stream;
  if (g.M <= 0 || g.N <= 0 || g.K <= 0 || g.batch <= 0) return 0;
  if (g.epi == EPI_NORM_BWD && (!g.aux || !g.out2 || !g.norm_part || !g.norm_r || g.n_npart <= 0))
    return 1;
  if (g.norm_part_out && (g.epi != EPI_DRELU2 || g.n_npart < (g.N + EC - 1) / EC)) return 1;
  if (g.fp8) {
    // e4m3 operands: K-major A and B (16-byte aligned rows), one product, the
    // dequantization factors given, no split; not the cross-entropy epilogues
    if (g.a_mn_major || g.b_mn_major || g.batch != 1 || !g.a_row_scale || !g.b_scale ||
        (g.lda | g.ldb) % 16 || g.epi == EPI_CE_FWD || g.epi == EPI_CE_BWD)
      return 1;
    const int tiles = ((g.M + P_BM - 1) / P_BM) * ((g.N + BN - 1) / BN);
    const int pairs = num_sms() / 2;
    return launch_pair<false, false, true>(g, 2 * (tiles < pairs ? tiles : pairs), 1, st);
  }
  if (g.batch > 1) {
    // a partial K block would read the next product's rows; the other
    // epilogues are not batched
    if (g.K % BK || !((g.epi == EPI_STORE && !g.beta) || g.epi == EPI_AXPBY)) return 1;
    if (int64_t(g.batch) * std::max(g.a_bstride, g.b_bstride) + std::max(g.M, std::max(g.N, g.K)) >
        (int64_t(1) << 31))
      return 1;
  }
  const int tiles = ((g.M + P_BM - 1) / P_BM) * ((g.N + BN - 1) / BN) * g.batch;
  if (g.epi == EPI_CE_FWD) g.n_part = (g.N + EC - 1) / EC;
  const int splits = gemm_tc_splits(g);
  const int pairs = num_sms() / 2;
  const int units = tiles * splits;
  const int grid = 2 * (units < pairs ? units : pairs);
  int rc;
  if (!g.a_mn_major && !g.b_mn_major) rc = launch_pair<false, false>(g, grid, splits, st);
  else if (!g.a_mn_major && g.b_mn_major) rc = launch_pair<false, true>(g, grid, splits, st);
  else if (g.a_mn_major && g.b_mn_major) rc = launch_pair<true, true>(g, grid, splits, st);
  else rc = launch_pair<true, false>(g, grid, splits, st);
  if (rc || splits == 1) return rc;
  const int64_t n4 = int64_t(g.M) * g.N / 4;
  splitk_reduce_kernel<<<int((n4 + 255) / 256), 256, 0, st>>>(
      g.splitk, static_cast<__nv_bfloat16*>(g.out), n4, splits, g.beta);
  return last_launch_rc();
}

int gemm_tc_tile_n() { return EC; }

}  // namespace gpt
