// Internal declarations of libgpt: workspace layout and kernel launchers.
// Host-only C++ (no CUDA headers needed to include it).
#pragma once

#include <cstddef>
#include <cstdint>

#include "gpt.h"

namespace gpt {

// Columns of the [q | k | v] projection: n_head query heads and n_kv_head key
// and value heads of head_dim each (gpt_config_init sets n_kv_head).
inline int64_t qkv_cols(const gpt_config& c) {
  return int64_t(c.n_head + 2 * c.n_kv_head) * c.head_dim;
}
// The sliding window as a key-distance bound: query i sees keys j with
// i - j < window_span(c).  A window of T or more positions (or none) is the
// full causal window, so the span is capped at T, which also keeps the
// kernels' key and query bounds (position + span) far from int overflow.
inline int window_span(const gpt_config& c) {
  return c.attn_window > 0 && c.attn_window < c.seq_len ? c.attn_window : c.seq_len;
}

// Block variants.  Value embeddings on layers l % ve_every == ve_every - 1.
inline bool has_value_embed(const gpt_config& c, int l) {
  return c.ve_every > 0 && l % c.ve_every == c.ve_every - 1;
}
inline int backout_layer(const gpt_config& c) { return c.n_layer / 2; }
constexpr int kSmearChannels = 24;  // the smear gate reads x[:, :, :24]
inline bool has_variants(const gpt_config& c) {
  return c.ve_every > 0 || c.resid_lambdas || c.smear || c.backout;
}
int64_t base_param_elems(const gpt_config& c);
int64_t variant_walk(const gpt_config& c, int tensor, int layer, int64_t* at, int64_t* rows,
                     int64_t* cols, int64_t* count);

// Kernel ids recorded in gpt_device_status::where.
enum KernelId : int32_t {
  K_EMBED = 1,
  K_CE_MERGE = 2,
  K_GEMM_TC = 3,
  K_ATTN = 4,
  K_LOSS = 5,
  K_WAITCHECK = 6,
};

// Epilogues of the GEMM C[m,n] = sum_k A(m,k) B(n,k).
enum Epilogue : int32_t {
  EPI_STORE = 0,    // out_t[m*ldo+n] = acc (+ out_t if beta)
  EPI_STORE_F32,    // out_f32[m*ldo+n] = acc
  EPI_RESID_F32,    // out_f32[m*ldo+n] += acc        (residual stream update)
  EPI_RELU2,        // out_t = max(acc,0)^2           (MLP activation)
  EPI_DRELU2,       // out_t = acc * 2*sqrt(aux_t)    (ReLU^2' from the stored activation)
  EPI_CE_FWD,       // per-row partial (max, sum exp) over the tile's columns + target logit
  EPI_CE_BWD,       // out_t = (exp(acc - lse[m]) - [n == tgt[m]]) * inv_n; 0 for n >= n_valid
  EPI_QKV,          // [q|k|v] row: RoPE + per-head RMSNorm of q, k; head-major scatter of q, k, v
  EPI_AXPBY,        // out_t = alpha * acc + beta_aux * aux_t   (Newton-Schulz updates)
  EPI_NORM_BWD,     // RMSNorm backward of the GEMM's output row (see norm_* below):
                    // out_f32 += r[m] (acc - aux_t * s[m]); out2_t = bf16(out_f32)
};

struct GemmArgs {
  // operands; element (m,k) of A is A[m*lda+k] if !a_mn_major else A[k*lda+m]
  const void* A;
  const void* B;
  int64_t lda, ldb;
  bool a_mn_major, b_mn_major;
  int M, N, K;
  // epilogue
  Epilogue epi;
  void* out;
  int64_t ldo;
  int beta;                 // EPI_STORE: 1 = accumulate into out
  const void* aux;          // EPI_DRELU2, EPI_AXPBY: second input, leading dim ldo
  float alpha = 1.f, beta_aux = 0.f;  // EPI_AXPBY scales
  // cross-entropy epilogues
  const int32_t* targets;   // [M]
  float* part_max;          // [M, n_part]
  float* part_sum;          // [M, n_part]
  float* tgt_logit;         // [M]
  const float* lse;         // [M]
  int n_part;               // partial columns per row = ceil(N / tile_n)
  float inv_n;
  int n_valid;              // columns >= n_valid are padding (EPI_CE_BWD writes 0)
  int32_t* status;          // device status word
  // EPI_QKV (rows = tokens b*T + t, columns = [q | k | v]: n_head q heads,
  // then n_kv_head k heads and n_kv_head v heads, head_dim each)
  void* q_out;              // [B, n_head, T, hd]
  void* k_out;
  void* v_out;              // [B, n_kv_head, T, hd] each
  float* rq;                // [B, n_head, T]: 1/rms of the rotated q rows
  float* rk;                // [B, n_kv_head, T]: the same for k
  const float* rope_cos;
  const float* rope_sin;    // [hd/2, T]: position-contiguous, one table row per pair index
  int seq_len, n_head, head_dim, qk_norm;
  int n_kv_head;
  float norm_eps;
  // batched products (tensor-core GEMM; EPI_STORE without beta or EPI_AXPBY,
  // K a multiple of 64): product b reads A and B `a_bstride` / `b_bstride` rows
  // further down their stored arrays and writes out (and reads aux) `o_bstride`
  // rows further down
  int batch = 1;
  int64_t a_bstride = 0, b_bstride = 0, o_bstride = 0;
  // 8-bit operands (tensor-core GEMM, K-major A and B): A and B hold e4m3
  // codes; the epilogue first multiplies the accumulator of row m by
  // a_row_scale[m] * (*b_scale), the operands' dequantization factors
  bool fp8 = false;
  const float* a_row_scale = nullptr;
  const float* b_scale = nullptr;
  // RMSNorm backward folded into GEMM epilogues (tensor-core GEMM, bf16).
  // EPI_DRELU2 with norm_part_out: also writes, per row m and 128-column
  // block p of the output, norm_part_out[m * n_npart + p] = sum of acc * aux
  // over the block's columns (the accumulator before the ReLU^2' factor).
  // EPI_NORM_BWD: s[m] = norm_scale * sum_p norm_part[m * n_npart + p],
  // r[m] = norm_r[m]; out is the fp32 gradient it accumulates into, out2
  // (bf16, leading dim ldo) receives its rounded copy, aux holds the norm's
  // output h.
  float* norm_part_out = nullptr;
  const float* norm_part = nullptr;
  const float* norm_r = nullptr;
  void* out2 = nullptr;
  int n_npart = 0;
  float norm_scale = 0.f;
  // split-K (tensor-core GEMM, EPI_STORE only): fp32 partials [splits][M][N]
  float* splitk;
  int64_t splitk_floats;    // capacity of `splitk`
};

struct LayerOffsets {
  uint64_t h1, r1, q, k, v, rq, rk, o, lse, h2, r2, a;
};

// Byte offsets of every workspace region.  Computed from the config only.
struct Layout {
  int64_t N;               // batch * seq_len
  int64_t vpad;            // vocab rounded up to 256 (row stride of the logit-gradient buffer)
  int esz;                 // bytes per stored activation element (2 bf16, 4 f32)
  // RoPE tables [T, hd/2] and the same transposed, [hd/2, T]
  uint64_t status, tok_stage, tgt_stage, rope_cos, rope_sin, rope_cos_tr, rope_sin_tr;
  uint64_t x, dxs;
  uint64_t layer_base, layer_stride;
  LayerOffsets lo;         // offsets relative to the layer's base
  uint64_t hf, rf;
  uint64_t qkv_raw;
  uint64_t part_max, part_sum, tgt_logit, lse_z, tok_loss, loss_acc;
  uint64_t npart;          // [N, n_npart] fp32: the folded norm backwards' row partials
  int64_t n_npart;
  uint64_t G, dh, du, dO, dqkv, Dattn;
  uint64_t splitk;          // fp32 split-K partials
  int64_t splitk_floats;
  uint64_t sort_perm, sort_offs, sort_count, sort_tilehist, scat_items, scat_item_offs,
      scat_partial;
  int64_t n_part_max;      // partial-stat columns reserved per row
  int64_t sort_tiles;      // N / 1024 rounded up
  int64_t scat_max_items;  // upper bound of (row, chunk) work items of the scatter
  // optimizer scratch (bf16 configs): Newton-Schulz iterates, Gram matrices,
  // sum-of-squares partials
  uint64_t opt_x0, opt_x1, opt_a, opt_b, opt_part;
  uint64_t opt_rows;       // NorMuon per-row scratch: v_mean and factors [2][max rows]
  // e4m3 block projections (fp8 configs): weight codes at the parameter
  // buffer's element offsets (one byte each), their dequantization factors
  // and amax bits [4 kinds][n_layer], the codes of each W^T at the same
  // offsets (for the data gradients), one activation's or output gradient's
  // codes [N, max(d, F, q|k|v columns)] and its per-row factors [N]
  uint64_t w8, w8_deq, w8_amax, w8t, a8, a8_deq;
  // block variants: smear (embedding, gate values, step-1 results), residual
  // scaling (x0, every layer's pre-scaling stream, the x0 gradient), backout
  // (x_b, the final stream gradient), value embeddings (table-gradient rows,
  // gate gradients), reduction partials
  uint64_t emb, sm_sg, sm_dg, sm_du, x0, xprev, dx0, xb, dxf, ve_rows, ve_dgz, vred;
  uint64_t total;
};

bool make_layout(const gpt_config& c, Layout* L);

// ---- bounded-wait expiry check (csrc/waitcheck.cu) ----
int launch_wait_expiry(int32_t* status, uint64_t limit_ns, void* stream);

// ---- optimizer (csrc/optim.cu) ----
constexpr int kOptNormBlocks = 296;  // fixed grid of the deterministic sum of squares
int launch_optim_init(const void* params, float* master, float* m, float* v, int64_t n, void* stream);
int launch_quant_rows(const void* x, int64_t rows, int cols, void* q, float* deq, void* stream);
int launch_quant_tensors(const void* x, int64_t n, int64_t stride, int n_mat, void* q, float* deq,
                         unsigned* amax_bits, void* stream);
// codes of each W^T ([cols, rows]; rows, cols multiples of 64) with the scale
// of the amax bits launch_quant_tensors left for the same matrices
int launch_quant_tensors_t(const void* x, int rows, int cols, int64_t stride, int n_mat,
                           const unsigned* amax_bits, void* q, void* stream);
int launch_adamw(void* params, const void* grads, float* master, float* m, float* v, int64_t n,
                 float lr, float b1, float b2, float eps, float wd, float bc1, float bc2, void* stream);
// M = mu M + G; U = nesterov ? G + mu M : M; x = bf16(U / (||U||_F + 1e-7)).
// partial: kOptNormBlocks + 1 floats of scratch.
int launch_muon_prepare(const void* grads, float* mom, int64_t n, float mu, int nesterov,
                        float* partial, void* x_out, void* stream);
// master -= step * x; params = bf16(master)
int launch_muon_apply(const void* x, float* master, void* params, int64_t n, float step, void* stream);
// NorMuon row factors of one update x [rows, cols]: buf (per-row state) is
// updated; factor[r] = step_size[r] * v_norm / max(v_norm_new, 1e-10); vmean:
// rows floats of scratch
int launch_normuon(const void* x, float* buf, int rows, int cols, float beta2, float* vmean,
                   float* factor, void* stream);
// master -= step * factor[row] * x; params = bf16(master)
int launch_muon_apply_rows(const void* x, float* master, void* params, int rows, int cols,
                           float step, const float* factor, void* stream);

// ---- launchers (all enqueue on `stream`, return cudaError_t as int) ------
int launch_rope_table(const gpt_config& c, float* cos_t, float* sin_t, float* cos_tr, float* sin_tr,
                      void* stream);
int launch_embed_norm(const gpt_config& c, const int32_t* tok, const void* wte, float* x,
                      void* h, float* r, int32_t* status, void* stream);
int launch_rms_fwd(const gpt_config& c, const float* x, void* h, float* r, void* stream);
int launch_rms_bwd(const gpt_config& c, const void* dh, const void* h, const float* r,
                   float* dx, void* dxs, int accumulate, void* stream);
int launch_qkv_post(const gpt_config& c, const void* qkv_raw, const float* cos_t,
                    const float* sin_t, void* q, void* k, void* v, float* rq, float* rk,
                    void* stream);
int launch_ce_merge(const gpt_config& c, const float* part_max, const float* part_sum,
                    int n_part, const float* tgt_logit, const int32_t* targets, float* lse,
                    float* tok_loss, int32_t* status, void* stream);
int launch_loss_mean(const gpt_config& c, const float* tok_loss, float* loss,
                     float* user_tok_loss, int32_t* status, void* stream);
int launch_attn_fwd(const gpt_config& c, const void* q, const void* k, const void* v, void* o,
                    float* lse, int32_t* status, void* stream);
// norm_part (bf16 only, or null): per token b*T + t, row stride H + 2*Hkv,
// each q head's, then k head's, then v head's share of sum_c dqkv_c * qkv_c,
// qkv the QKV projection's raw output (for the backward of the norm before it)
int launch_attn_bwd(const gpt_config& c, const void* q, const void* k, const void* v,
                    const void* o, const void* dO, const float* lse, const float* rq,
                    const float* rk, const float* cos_t, const float* sin_t, float* Dbuf,
                    void* dqkv, float* norm_part, int32_t* status, void* stream);
int launch_sort_tokens(const gpt_config& c, const Layout& L, const int32_t* tok, char* ws,
                       void* stream);
int launch_embed_scatter(const gpt_config& c, const Layout& L, const float* dx0, char* ws,
                         void* dwte, int accumulate, void* stream);
// ---- block variants (csrc/variants.cu) ----
int launch_smear_fwd(const gpt_config& c, const float* e, const void* w, const void* scalars, float* x,
                     float* sg, void* stream);
int launch_lambda_mix(const gpt_config& c, float* x, const float* x0, float* xprev, const void* lam,
                      void* stream);
int launch_axpy(const gpt_config& c, float* y, const float* x, const void* s, float mul, void* stream);
int launch_ve_fwd(const gpt_config& c, const void* h, const void* wg, const void* ve, const int32_t* tok,
                  void* v, void* stream);
int launch_ve_bwd(const gpt_config& c, const void* dqkv, const void* h, const void* wg, const void* ve,
                  const int32_t* tok, float* rows, float* dgz, void* d_wg, int accumulate, void* stream);
int launch_ve_dh(const gpt_config& c, void* dh, const float* dgz, const void* wg, void* stream);
int launch_resid_bwd(const gpt_config& c, float* dx, void* dxs, const float* dxf, const void* scalars,
                     const float* xprev, const float* x0, float* dx0, const void* lam, float* partial,
                     void* d_lam, int accumulate, void* stream);
int launch_dot(const gpt_config& c, const float* x, const float* y, float scale, float* partial,
               void* out, int accumulate, void* stream);
int launch_smear_bwd(const gpt_config& c, const float* dx, float* e, const float* sg, float* dg,
                     float* du, const void* w, const void* scalars, void* d_w, void* d_scalars,
                     int accumulate, void* stream);
int variant_red_floats();

int launch_gemm(const gpt_config& c, const GemmArgs& g, void* stream);
// Number of kernels launch_gemm enqueues for these arguments (2 with a split-K reduce).
int gemm_kernel_count(const gpt_config& c, const GemmArgs& g);
// Column width of the GEMM tile that produces the logits (partial-statistics granularity).
int gemm_ce_tile_n(const gpt_config& c);

}  // namespace gpt
