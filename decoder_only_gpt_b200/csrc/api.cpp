// libgpt C ABI: configuration, parameter / workspace layout and the step
// orchestration (which kernel runs when, on which buffers).  Every numeric
// step runs in the CUDA kernels of this directory; this file only enqueues.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <vector>

#include "gpt_internal.h"
#include "trace.h"

namespace gpt {
namespace {

constexpr uint64_t kAlign = 256;

uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

struct Bump {
  uint64_t off = 0;
  uint64_t take(uint64_t bytes) {
    off = align_up(off, kAlign);
    uint64_t o = off;
    off += bytes;
    return o;
  }
};

int64_t param_elems_aligned(int64_t n) { return (n + 127) / 128 * 128; }


bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? GPT_OK : GPT_ECUDA; }

#define GPT_TRY(expr)                           \
  do {                                          \
    int rc_ = (expr);                           \
    if (rc_ != 0) return rc_ > 0 ? GPT_ECUDA : rc_; \
  } while (0)

}  // namespace

// Elements of the base model's parameters (wte, the layers, lm_head), aligned.
int64_t base_param_elems(const gpt_config& c) {
  const int64_t d = c.d_model, F = c.d_ff, V = c.vocab, Q = qkv_cols(c);
  return 2 * param_elems_aligned(V * d) +
         int64_t(c.n_layer) * (param_elems_aligned(Q * d) + param_elems_aligned(d * d) +
                               2 * param_elems_aligned(F * d));
}

// Walk the block-variant tensors in their buffer order (after lm_head): for
// each value-embedding layer its table and gate, then the residual scales,
// the smear gate, the scalars.  Returns the aligned element count of all of
// them; finds (tensor, layer)'s offset from the variants' start (at, rows,
// cols; at stays -1 when absent) and adds the unaligned count to *count.
int64_t variant_walk(const gpt_config& c, int tensor, int layer, int64_t* at, int64_t* rows,
                     int64_t* cols, int64_t* count) {
  int64_t off = 0;
  auto take = [&](int t, int l, int64_t r, int64_t cc) {
    if (t == tensor && (l == layer || (t != GPT_T_VE && t != GPT_T_VE_GATE))) {
      *at = off;
      *rows = r;
      *cols = cc;
    }
    if (count) *count += r * cc;
    off += param_elems_aligned(r * cc);
  };
  const int64_t kvd = int64_t(c.n_kv_head ? c.n_kv_head : c.n_head) * c.head_dim;
  for (int l = 0; l < c.n_layer; ++l)
    if (has_value_embed(c, l)) {
      take(GPT_T_VE, l, c.vocab, kvd);
      take(GPT_T_VE_GATE, l, c.n_kv_head ? c.n_kv_head : c.n_head, c.ve_gate_channels);
    }
  if (c.resid_lambdas) take(GPT_T_LAMBDAS, 0, c.n_layer, 2);
  if (c.smear) take(GPT_T_SMEAR_GATE, 0, 1, kSmearChannels);
  if (c.smear || c.backout) take(GPT_T_SCALARS, 0, 1, 2);
  return off;
}

bool make_layout(const gpt_config& c, Layout* L) {
  const int64_t N = int64_t(c.batch) * c.seq_len;
  const int64_t d = c.d_model, F = c.d_ff, V = c.vocab, H = c.n_head, T = c.seq_len,
                B = c.batch, hd = c.head_dim, Hkv = c.n_kv_head, dkv = Hkv * hd, Q = qkv_cols(c);
  const int esz = c.dtype == GPT_BF16 ? 2 : 4;
  L->N = N;
  L->esz = esz;
  L->vpad = (V + 255) / 256 * 256;
  Bump b;
  L->status = b.take(sizeof(gpt_device_status) < 256 ? 256 : sizeof(gpt_device_status));
  L->tok_stage = b.take(N * 4);
  L->tgt_stage = b.take(N * 4);
  L->rope_cos = b.take(T * (hd / 2) * 4);
  L->rope_sin = b.take(T * (hd / 2) * 4);
  L->rope_cos_tr = b.take(T * (hd / 2) * 4);
  L->rope_sin_tr = b.take(T * (hd / 2) * 4);
  L->x = b.take(N * d * 4);
  L->dxs = b.take(N * d * esz);
  // one layer's saved activations
  Bump lb;
  L->lo.h1 = lb.take(N * d * esz);
  L->lo.r1 = lb.take(N * 4);
  L->lo.q = lb.take(N * d * esz);
  L->lo.k = lb.take(N * dkv * esz);
  L->lo.v = lb.take(N * dkv * esz);
  L->lo.rq = lb.take(B * H * T * 4);
  L->lo.rk = lb.take(B * Hkv * T * 4);
  L->lo.o = lb.take(N * d * esz);
  L->lo.lse = lb.take(B * H * T * 4);
  L->lo.h2 = lb.take(N * d * esz);
  L->lo.r2 = lb.take(N * 4);
  L->lo.a = lb.take(N * F * esz);
  L->layer_stride = align_up(lb.off, kAlign);
  // optimizer scratch (bf16), in the same bytes as the saved activations (dead
  // once gpt_backward has run): for every layer, two Newton-Schulz iterates of
  // the largest block matrix and two Gram matrices of the smaller side (d for
  // every block matrix), so that one kind of matrix is orthogonalised for all
  // layers at once
  uint64_t opt_bytes = 0;
  if (c.dtype == GPT_BF16) {
    const int64_t mat = std::max(std::max(Q * d, F * d), d * d);
    const int64_t gd = d;  // Wqkv is [Q, d] with Q >= d, Wup [F, d], Wdown [d, F], Wo [d, d]
    Bump ob;
    L->opt_x0 = ob.take(mat * 2 * c.n_layer);
    L->opt_x1 = ob.take(mat * 2 * c.n_layer);
    L->opt_a = ob.take(gd * gd * 2 * c.n_layer);
    L->opt_b = ob.take(gd * gd * 2 * c.n_layer);
    opt_bytes = ob.off;
  }
  L->layer_base = b.take(std::max(L->layer_stride * uint64_t(c.n_layer), opt_bytes));
  L->hf = b.take(N * d * esz);
  L->rf = b.take(N * 4);
  L->qkv_raw = b.take(c.dtype == GPT_F32 ? N * Q * esz : 0);  // bf16: fused into the GEMM
  // cross-entropy partials: the narrowest GEMM tile used for the logits is 64 columns
  L->n_part_max = (V + 63) / 64;
  L->part_max = b.take(N * L->n_part_max * 4);
  L->part_sum = b.take(N * L->n_part_max * 4);
  L->tgt_logit = b.take(N * 4);
  L->lse_z = b.take(N * 4);
  L->tok_loss = b.take(N * 4);
  L->loss_acc = b.take(256);
  // the block norms' backward, folded into the data-gradient GEMMs (bf16): one
  // fp32 row partial per down-projection dgrad column block of >= 64, or per
  // attention head (q, k and v heads)
  L->n_npart = std::max((F + 63) / 64, H + 2 * Hkv);
  L->npart = b.take(c.dtype == GPT_BF16 ? N * L->n_npart * 4 : 0);
  L->G = b.take(N * L->vpad * esz);
  L->dh = b.take(N * d * esz);
  L->du = b.take(N * F * esz);
  L->dO = b.take(N * d * esz);
  L->dqkv = b.take(N * Q * esz);
  L->Dattn = b.take(B * H * T * 4);
  // split-K partials of the weight-gradient GEMMs (up to 4 splits of the largest layer matrix)
  L->splitk_floats = c.dtype == GPT_BF16 ? 4 * std::max(std::max(Q * d, F * d), d * d) : 0;
  L->splitk = b.take(L->splitk_floats * 4);
  // deterministic embedding scatter
  L->sort_tiles = (N + 1023) / 1024;
  L->sort_perm = b.take(N * 4);
  L->sort_offs = b.take((V + 1) * 4);
  L->sort_count = b.take((V + 1) * 4);
  L->sort_tilehist = b.take(L->sort_tiles * V * 4);
  L->scat_max_items = N / 64 + V + 1;
  L->scat_items = b.take(L->scat_max_items * 8);
  L->scat_item_offs = b.take((V + 1) * 8);
  L->scat_partial = b.take((N / 64 + 1) * d * 4 * 2);
  // e4m3 forward projections
  if (c.fp8) {
    L->w8 = b.take(uint64_t(c.param_bytes / 2));
    L->w8_deq = b.take(4 * uint64_t(c.n_layer) * 4);
    L->w8_amax = b.take(4 * uint64_t(c.n_layer) * 4);
    L->w8t = b.take(uint64_t(c.param_bytes / 2));
    L->a8 = b.take(N * std::max(std::max(d, F), int64_t(qkv_cols(c))));
    L->a8_deq = b.take(N * 4);
  } else {
    L->w8 = L->w8_deq = L->w8_amax = L->w8t = L->a8 = L->a8_deq = 0;
  }
  // block variants
  {
    const int64_t nd4 = N * d * 4, Hkv = c.n_kv_head ? c.n_kv_head : c.n_head;
    bool any_ve = false;
    for (int l = 0; l < c.n_layer; ++l) any_ve |= has_value_embed(c, l);
    L->emb = c.smear ? b.take(nd4) : 0;
    L->sm_sg = c.smear ? b.take(N * 4) : 0;
    L->sm_dg = c.smear ? b.take(N * 4) : 0;
    L->sm_du = c.smear ? b.take(N * 4) : 0;
    L->x0 = c.resid_lambdas ? b.take(nd4) : 0;
    L->xprev = c.resid_lambdas ? b.take(nd4 * c.n_layer) : 0;
    L->dx0 = c.resid_lambdas ? b.take(nd4) : 0;
    L->xb = c.backout ? b.take(nd4) : 0;
    L->dxf = c.backout ? b.take(nd4) : 0;
    L->ve_rows = any_ve ? b.take(N * Hkv * c.head_dim * 4) : 0;
    L->ve_dgz = any_ve ? b.take(N * Hkv * 4) : 0;
    L->vred = has_variants(c) ? b.take(int64_t(variant_red_floats()) * 4) : 0;
  }
  // Muon's sum-of-squares partials and reciprocal norm
  if (c.dtype == GPT_BF16) {
    L->opt_x0 += L->layer_base;
    L->opt_x1 += L->layer_base;
    L->opt_a += L->layer_base;
    L->opt_b += L->layer_base;
    L->opt_part = b.take((kOptNormBlocks + 1) * 4);
    L->opt_rows = b.take(2 * std::max(std::max(Q, F), d) * 4);
  } else {
    L->opt_x0 = L->opt_x1 = L->opt_a = L->opt_b = L->opt_part = L->opt_rows = 0;
  }
  L->total = align_up(b.off, kAlign);
  return true;
}

}  // namespace gpt

using namespace gpt;

extern "C" {

const char* gpt_version(void) { return "libgpt 0.1 (sm_100a)"; }

const char* gpt_strerror(int code) {
  switch (code) {
    case GPT_OK: return "ok";
    case GPT_EINVAL: return "invalid argument (null, misaligned or inconsistent)";
    case GPT_EUNSUPPORTED: return "unsupported shape or dtype";
    case GPT_ECUDA: return "CUDA call failed";
    case GPT_EDATA: return "token or target id outside [0, vocab)";
    case GPT_ETIMEOUT: return "bounded device wait expired";
    case GPT_ENONFINITE: return "loss is not finite";
    default: return "unknown error code";
  }
}

int gpt_config_init(gpt_config* c) {
  if (!c) return GPT_EINVAL;
  if (c->rope_base == 0.f) c->rope_base = 10000.f;
  if (c->norm_eps == 0.f) c->norm_eps = 1e-6f;
  if (c->n_kv_head == 0) c->n_kv_head = c->n_head;
  if (c->n_layer < 0 || c->d_model <= 0 || c->n_head <= 0 || c->head_dim <= 0 ||
      c->d_ff <= 0 || c->vocab < 2 || c->seq_len <= 0 || c->batch <= 0)
    return GPT_EINVAL;
  if (int64_t(c->n_head) * c->head_dim != c->d_model) return GPT_EINVAL;
  if (c->n_kv_head <= 0 || c->n_head % c->n_kv_head || c->attn_window < 0) return GPT_EINVAL;
  if (c->fp8 != 0 && c->fp8 != 1) return GPT_EINVAL;
  if (c->fp8 && c->dtype != GPT_BF16) return GPT_EUNSUPPORTED;
  if (!(c->rope_base > 1.f) || !(c->norm_eps > 0.f) || !std::isfinite(c->rope_base) ||
      !std::isfinite(c->norm_eps))
    return GPT_EINVAL;
  if (c->qk_norm != 0 && c->qk_norm != 1) return GPT_EINVAL;
  if (c->dtype == GPT_BF16) {
    if (c->d_model % 64 || c->d_ff % 64) return GPT_EUNSUPPORTED;
    if (c->head_dim != 64 && c->head_dim != 128) return GPT_EUNSUPPORTED;
  } else if (c->dtype == GPT_F32) {
    if (c->head_dim % 2 || c->head_dim > 128) return GPT_EUNSUPPORTED;
    if (c->seq_len > 4096) return GPT_EUNSUPPORTED;
  } else {
    return GPT_EINVAL;
  }
  if (c->ve_every < 0 || (c->resid_lambdas != 0 && c->resid_lambdas != 1) ||
      (c->smear != 0 && c->smear != 1) || (c->backout != 0 && c->backout != 1))
    return GPT_EINVAL;
  if (c->ve_every > 0 && c->ve_gate_channels == 0) c->ve_gate_channels = std::min(32, c->d_model);
  if (c->ve_every > 0 && (c->ve_gate_channels < 1 || c->ve_gate_channels > c->d_model)) return GPT_EINVAL;
  if (c->smear && c->d_model < kSmearChannels) return GPT_EUNSUPPORTED;
  if (c->backout && c->n_layer < 1) return GPT_EINVAL;
  const int64_t N = int64_t(c->batch) * c->seq_len;
  if (N > (int64_t(1) << 31) / 4 || int64_t(c->vocab) > (int64_t(1) << 24)) return GPT_EUNSUPPORTED;
  const int64_t d = c->d_model, F = c->d_ff, V = c->vocab, Q = qkv_cols(*c);
  int64_t n = 2 * V * d + int64_t(c->n_layer) * (Q * d + d * d + 2 * F * d);
  int64_t vn = 0;
  const int64_t elems = base_param_elems(*c) + variant_walk(*c, -1, -1, nullptr, nullptr, nullptr, &vn);
  c->n_params = n + vn;
  c->param_bytes = uint64_t(elems) * (c->dtype == GPT_BF16 ? 2 : 4);
  Layout L;
  make_layout(*c, &L);
  c->workspace_bytes = L.total;
  return GPT_OK;
}

int gpt_config_from_depth(gpt_config* c, int depth, int seq_len, int batch, int vocab) {
  if (!c || depth < 2 || depth % 2) return GPT_EINVAL;
  std::memset(c, 0, sizeof(*c));
  c->n_layer = depth;
  c->d_model = 64 * depth;
  c->head_dim = 128;
  c->n_head = c->d_model / 128;
  c->d_ff = 4 * c->d_model;
  c->vocab = vocab;
  c->seq_len = seq_len;
  c->batch = batch;
  c->dtype = GPT_BF16;
  c->qk_norm = 1;
  c->rope_base = 10000.f;
  c->norm_eps = 1e-6f;
  return gpt_config_init(c);
}

int gpt_param_offset(const gpt_config* c, int tensor, int layer, int64_t* off, int64_t* rows,
                     int64_t* cols) {
  if (!c || !off || !rows || !cols) return GPT_EINVAL;
  if (tensor >= GPT_T_VE && tensor <= GPT_T_SCALARS) {
    *off = -1;
    const int64_t o = base_param_elems(*c) + 0;
    int64_t r = 0, cc = 0, at = -1;
    variant_walk(*c, tensor, layer, &at, &r, &cc, nullptr);
    if (at < 0) return GPT_EINVAL;  // not present in this config (or no such layer)
    *off = o + at;
    *rows = r;
    *cols = cc;
    return GPT_OK;
  }
  const int64_t d = c->d_model, F = c->d_ff, V = c->vocab, Q = qkv_cols(*c);
  const bool per_layer = tensor >= GPT_T_WQKV && tensor <= GPT_T_WDOWN;
  if (tensor < GPT_T_WTE || tensor > GPT_T_LM_HEAD) return GPT_EINVAL;
  if (per_layer && (layer < 0 || layer >= c->n_layer)) return GPT_EINVAL;
  const int64_t lsz = param_elems_aligned(Q * d) + param_elems_aligned(d * d) +
                      2 * param_elems_aligned(F * d);
  const int64_t base = param_elems_aligned(V * d);
  switch (tensor) {
    case GPT_T_WTE: *off = 0; *rows = V; *cols = d; break;
    case GPT_T_WQKV: *off = base + layer * lsz; *rows = Q; *cols = d; break;
    case GPT_T_WO:
      *off = base + layer * lsz + param_elems_aligned(Q * d); *rows = d; *cols = d; break;
    case GPT_T_WUP:
      *off = base + layer * lsz + param_elems_aligned(Q * d) + param_elems_aligned(d * d);
      *rows = F; *cols = d; break;
    case GPT_T_WDOWN:
      *off = base + layer * lsz + param_elems_aligned(Q * d) + param_elems_aligned(d * d) +
             param_elems_aligned(F * d);
      *rows = d; *cols = F; break;
    case GPT_T_LM_HEAD: *off = base + int64_t(c->n_layer) * lsz; *rows = V; *cols = d; break;
  }
  return GPT_OK;
}

int gpt_workspace_region(const gpt_config* c, int region, int layer, uint64_t* off,
                         uint64_t* bytes) {
  if (!c || !off || !bytes) return GPT_EINVAL;
  Layout L;
  make_layout(*c, &L);
  const uint64_t N = L.N, d = c->d_model, V = c->vocab;
  switch (region) {
    case GPT_W_STATUS: *off = L.status; *bytes = sizeof(gpt_device_status); break;
    case GPT_W_RESID: *off = L.x; *bytes = N * d * 4; break;
    case GPT_W_LSE: *off = L.lse_z; *bytes = N * 4; break;
    case GPT_W_SORT_PERM: *off = L.sort_perm; *bytes = N * 4; break;
    case GPT_W_SORT_OFFS: *off = L.sort_offs; *bytes = (V + 1) * 4; break;
    case GPT_W_ATTN_LSE:
      if (layer < 0 || layer >= c->n_layer) return GPT_EINVAL;
      *off = L.layer_base + L.layer_stride * layer + L.lo.lse;
      *bytes = uint64_t(c->batch) * c->n_head * c->seq_len * 4;
      break;
    default: return GPT_EINVAL;
  }
  return GPT_OK;
}

static int check_common(const gpt_config* c, const int32_t* tok, const int32_t* tgt,
                        const void* params, void* ws) {
  if (!c || !tok || !tgt || !params || !ws) return GPT_EINVAL;
  gpt_config chk = *c;
  int rc = gpt_config_init(&chk);
  if (rc != GPT_OK) return rc;
  if (chk.param_bytes != c->param_bytes || chk.workspace_bytes != c->workspace_bytes)
    return GPT_EINVAL;  // derived fields stale: call gpt_config_init again
  if (!aligned(tok, 16) || !aligned(tgt, 16) || !aligned(params, 256) || !aligned(ws, 256))
    return GPT_EINVAL;
  return GPT_OK;
}



static GemmArgs gemm_kk(const void* A, int64_t lda, const void* B, int64_t ldb, int M, int N,
                        int K, Epilogue epi, void* out, int64_t ldo, int32_t* status) {
  GemmArgs g{};
  g.A = A; g.B = B; g.lda = lda; g.ldb = ldb;
  g.a_mn_major = false; g.b_mn_major = false;
  g.M = M; g.N = N; g.K = K; g.epi = epi; g.out = out; g.ldo = ldo;
  g.status = status;
  return g;
}

// Weight-gradient GEMMs get the workspace's split-K buffer (used when the tile
// count alone would leave SMs idle).
static GemmArgs with_splitk(GemmArgs g, const Layout& L, char* ws) {
  g.splitk = reinterpret_cast<float*>(ws + L.splitk);
  g.splitk_floats = L.splitk_floats;
  return g;
}

// ---- traced launch wrappers: algorithmic FLOPs / HBM bytes per launch -------
static int run_gemm(const gpt_config& c, const GemmArgs& g, cudaStream_t st) {
  const double e = c.dtype == GPT_BF16 ? 2.0 : 4.0;
  double bytes = (double(g.M) * g.K + double(g.N) * g.K) * (g.fp8 ? 1.0 : e);
  const double mn = double(g.M) * g.N;
  switch (g.epi) {
    case EPI_STORE: bytes += mn * e * (g.beta ? 2 : 1); break;
    case EPI_RESID_F32: bytes += mn * 8; break;
    case EPI_DRELU2: bytes += mn * e * 2 + (g.norm_part_out ? double(g.M) * g.n_npart * 4 : 0.0); break;
    case EPI_NORM_BWD: bytes += mn * (2 * e + 8) + double(g.M) * (g.n_npart + 1) * 4; break;
    case EPI_AXPBY: bytes += mn * e * 2; break;
    case EPI_CE_FWD: bytes += double(g.M) * 12; break;
    case EPI_QKV: bytes += mn * e + double(g.M) * (g.n_head + g.n_kv_head) * 4; break;
    default: bytes += mn * e; break;
  }
  TraceScope ts(GPT_K_GEMM, gemm_kernel_count(c, g), 2.0 * double(g.M) * g.N * g.K * g.batch,
                bytes * g.batch, st);
  return launch_gemm(c, g, st);
}

static double attn_pairs(const gpt_config& c) {  // visible (query, key) pairs
  const double T = c.seq_len, W = std::min<double>(window_span(c), T);
  return double(c.batch) * c.n_head * (W * T - W * (W - 1) / 2);
}

struct Step {
  const gpt_config* c;
  char* ws;
  const char* p;
  Layout L;
  int esz;
  int N, d, F, V;
  cudaStream_t st;
  int32_t* status;
  float* cos_t;
  float* sin_t;
  float* x;

  Step(const gpt_config* cfg, void* workspace, const void* params, void* stream) : c(cfg) {
    ws = static_cast<char*>(workspace);
    p = static_cast<const char*>(params);
    make_layout(*c, &L);
    esz = L.esz;
    N = int(L.N); d = c->d_model; F = c->d_ff; V = c->vocab;
    st = static_cast<cudaStream_t>(stream);
    status = reinterpret_cast<int32_t*>(ws + L.status);
    cos_t = reinterpret_cast<float*>(ws + L.rope_cos);
    sin_t = reinterpret_cast<float*>(ws + L.rope_sin);
    x = reinterpret_cast<float*>(ws + L.x);
  }
  char* layer(int l) const { return ws + L.layer_base + L.layer_stride * uint64_t(l); }
  float* f(uint64_t off) const { return reinterpret_cast<float*>(ws + off); }
  const void* param(int t, int l) const {
    int64_t off, r, cc;
    gpt_param_offset(c, t, l, &off, &r, &cc);
    return p + off * esz;
  }
  double nd() const { return double(N) * d; }

  // fp8 configs: e4m3 codes of every block matrix (per-tensor scales), once
  // per forward, from the bf16 parameters
  int quant_weights() {
    for (int kind = 0; kind < 4; ++kind) {
      const int tensor = GPT_T_WQKV + kind;
      int64_t off0, r, cc, off1 = 0;
      gpt_param_offset(c, tensor, 0, &off0, &r, &cc);
      if (c->n_layer > 1) gpt_param_offset(c, tensor, 1, &off1, &r, &cc);
      const int64_t stride = c->n_layer > 1 ? off1 - off0 : 0;
      TraceScope ts(GPT_K_QUANT, 3, 0, double(c->n_layer) * r * cc * 5, st);
      const int rc = launch_quant_tensors(p + off0 * esz, r * cc, stride, c->n_layer, ws + L.w8 + off0,
                                          f(L.w8_deq) + kind * c->n_layer,
                                          reinterpret_cast<unsigned*>(ws + L.w8_amax) + kind * c->n_layer,
                                          st);
      if (rc) return rc;
    }
    return 0;
  }
  // fp8 configs: the codes of every block matrix's transpose, for the data
  // gradients, with the scales the forward's quant_weights found
  int quant_weights_t() {
    for (int kind = 0; kind < 4; ++kind) {
      const int tensor = GPT_T_WQKV + kind;
      int64_t off0, r, cc, off1 = 0;
      gpt_param_offset(c, tensor, 0, &off0, &r, &cc);
      if (c->n_layer > 1) gpt_param_offset(c, tensor, 1, &off1, &r, &cc);
      const int64_t stride = c->n_layer > 1 ? off1 - off0 : 0;
      TraceScope ts(GPT_K_QUANT, 1, 0, double(c->n_layer) * r * cc * 3, st);
      const int rc = launch_quant_tensors_t(p + off0 * esz, int(r), int(cc), stride, c->n_layer, 
                                            reinterpret_cast<unsigned*>(ws + L.w8_amax) + kind * c->n_layer,
                                            ws + L.w8t + off0, st);
      if (rc) return rc;
    }
    return 0;
  }
  // the data gradient dX = dY W of block matrix `tensor` of layer l, given as
  // the bf16 GEMM (A = dY [N, K] K-major, B = W as the MN-major [K, N]); fp8
  // configs quantize dY per row and multiply it with the codes of W^T
  int dgrad(GemmArgs g, int tensor, int l) {
    if (!c->fp8) return run_gemm(*c, g, st);
    {
      TraceScope ts(GPT_K_QUANT, 1, 0, double(N) * g.K * 3 + N * 4.0, st);
      const int rc = launch_quant_rows(g.A, N, g.K, ws + L.a8, f(L.a8_deq), st);
      if (rc) return rc;
    }
    int64_t off, r, cc;
    gpt_param_offset(c, tensor, l, &off, &r, &cc);
    g.A = ws + L.a8;
    g.B = ws + L.w8t + off;
    g.lda = g.ldb = g.K;
    g.b_mn_major = false;
    g.fp8 = true;
    g.a_row_scale = f(L.a8_deq);
    g.b_scale = f(L.w8_deq) + (tensor - GPT_T_WQKV) * c->n_layer + l;
    return run_gemm(*c, g, st);
  }
  // fp8 configs: one block projection of the bf16 activation `xact` [N, K]:
  // quantize it per row into the scratch codes, then the e4m3 GEMM against the
  // weight's codes; otherwise the bf16 GEMM as given
  int projection(GemmArgs g, int tensor, int l) {
    if (!c->fp8) return run_gemm(*c, g, st);
    {
      TraceScope ts(GPT_K_QUANT, 1, 0, double(N) * g.K * 3 + N * 4.0, st);
      const int rc = launch_quant_rows(g.A, N, g.K, ws + L.a8, f(L.a8_deq), st);
      if (rc) return rc;
    }
    int64_t off, r, cc;
    gpt_param_offset(c, tensor, l, &off, &r, &cc);
    g.A = ws + L.a8;
    g.B = ws + L.w8 + off;
    g.lda = g.ldb = g.K;
    g.fp8 = true;
    g.a_row_scale = f(L.a8_deq);
    g.b_scale = f(L.w8_deq) + (tensor - GPT_T_WQKV) * c->n_layer + l;
    return run_gemm(*c, g, st);
  }

  int rms_fwd(void* h, float* r) {
    TraceScope ts(GPT_K_NORM, 1, 0, nd() * (4 + esz) + N * 4.0, st);
    return launch_rms_fwd(*c, x, h, r, st);
  }
  int rms_bwd(const void* dh, const void* h, const float* r, int acc) {
    TraceScope ts(GPT_K_NORM, 1, 0, nd() * (2 * esz + (acc ? 4 : 0) + 4 + esz) + N * 4.0, st);
    return launch_rms_bwd(*c, dh, h, r, x, ws + L.dxs, acc, st);
  }
};

int gpt_forward_loss(const gpt_config* c, const int32_t* tok, const int32_t* tgt,
                     const void* params, void* workspace, float* loss, float* token_loss,
                     void* stream) {
  int rc = check_common(c, tok, tgt, params, workspace);
  if (rc) return rc;
  if (!loss || !aligned(loss, 4) || (token_loss && !aligned(token_loss, 4))) return GPT_EINVAL;
  Step S(c, workspace, params, stream);
  const Layout& L = S.L;
  const int N = S.N, d = S.d, F = S.F, V = S.V, esz = S.esz;
  char* ws = S.ws;
  cudaStream_t st = S.st;
  {
    TraceScope ts(GPT_K_OTHER, 2, 0, c->seq_len * c->head_dim * 4.0, st);
    GPT_TRY(cuda_rc(cudaMemsetAsync(ws + L.status, 0, 256, st)));
    GPT_TRY(launch_rope_table(*c, S.cos_t, S.sin_t, reinterpret_cast<float*>(ws + L.rope_cos_tr),
                              reinterpret_cast<float*>(ws + L.rope_sin_tr), st));
  }
  {
    void* h0 = c->n_layer > 0 ? (void*)(S.layer(0) + L.lo.h1) : (void*)(ws + L.hf);
    float* r0 = reinterpret_cast<float*>(c->n_layer > 0 ? S.layer(0) + L.lo.r1 : ws + L.rf);
    TraceScope ts(GPT_K_NORM, 1, 0, S.nd() * (esz + 4 + esz) + N * 8.0, st);
    GPT_TRY(launch_embed_norm(*c, tok, S.param(GPT_T_WTE, 0), S.x, h0, r0, S.status, st));
  }
  const uint64_t nd4 = uint64_t(N) * d * 4;
  if (c->smear) {  // x = e + s sigmoid(e[:24] . w) e_prev, from a copy of the gathered e
    TraceScope ts(GPT_K_OTHER, 2, 0, S.nd() * 16.0, st);
    GPT_TRY(cuda_rc(cudaMemcpyAsync(ws + L.emb, S.x, nd4, cudaMemcpyDeviceToDevice, st)));
    GPT_TRY(launch_smear_fwd(*c, S.f(L.emb), S.param(GPT_T_SMEAR_GATE, 0), S.param(GPT_T_SCALARS, 0), S.x,
                             S.f(L.sm_sg), st));
    if (c->n_layer == 0) GPT_TRY(S.rms_fwd(ws + L.hf, S.f(L.rf)));
  }
  if (c->resid_lambdas) {  // x0: the stream entering layer 0
    TraceScope ts(GPT_K_OTHER, 1, 0, S.nd() * 8.0, st);
    GPT_TRY(cuda_rc(cudaMemcpyAsync(ws + L.x0, S.x, nd4, cudaMemcpyDeviceToDevice, st)));
  }
  const double attn_f = 4.0 * attn_pairs(*c) * c->head_dim;  // QK^T and PV, visible pairs
  const int Qc = int(qkv_cols(*c));
  if (c->fp8 && c->n_layer > 0) GPT_TRY(S.quant_weights());
  for (int l = 0; l < c->n_layer; ++l) {
    char* Lb = S.layer(l);
    {  // block variants at the layer's entry: residual scaling, the backout point
      bool renorm = l == 0 && c->smear;
      if (c->resid_lambdas) {
        TraceScope ts(GPT_K_OTHER, 1, 0, S.nd() * 16.0, st);
        const char* lam = static_cast<const char*>(S.param(GPT_T_LAMBDAS, 0)) + int64_t(l) * 2 * esz;
        GPT_TRY(launch_lambda_mix(*c, S.x, S.f(L.x0), S.f(L.xprev + uint64_t(l) * nd4), lam, st));
        renorm = true;
      }
      if (c->backout && l == backout_layer(*c)) {
        TraceScope ts(GPT_K_OTHER, 1, 0, S.nd() * 8.0, st);
        GPT_TRY(cuda_rc(cudaMemcpyAsync(ws + L.xb, S.x, nd4, cudaMemcpyDeviceToDevice, st)));
      }
      if (renorm) GPT_TRY(S.rms_fwd(Lb + L.lo.h1, reinterpret_cast<float*>(Lb + L.lo.r1)));
    }
    if (c->dtype == GPT_BF16) {
      // QKV projection with RoPE, QK-norm and the head-major scatter in its epilogue
      GemmArgs g = gemm_kk(Lb + L.lo.h1, d, S.param(GPT_T_WQKV, l), d, N, Qc, d, EPI_QKV,
                           nullptr, Qc, S.status);
      g.q_out = Lb + L.lo.q; g.k_out = Lb + L.lo.k; g.v_out = Lb + L.lo.v;
      g.rq = reinterpret_cast<float*>(Lb + L.lo.rq);
      g.rk = reinterpret_cast<float*>(Lb + L.lo.rk);
      g.rope_cos = reinterpret_cast<const float*>(ws + L.rope_cos_tr);
      g.rope_sin = reinterpret_cast<const float*>(ws + L.rope_sin_tr);
      g.seq_len = c->seq_len; g.n_head = c->n_head; g.head_dim = c->head_dim;
      g.n_kv_head = c->n_kv_head;
      g.qk_norm = c->qk_norm; g.norm_eps = c->norm_eps;
      GPT_TRY(S.projection(g, GPT_T_WQKV, l));
    } else {
      GPT_TRY(run_gemm(*c, gemm_kk(Lb + L.lo.h1, d, S.param(GPT_T_WQKV, l), d, N, Qc, d,
                                   EPI_STORE, ws + L.qkv_raw, Qc, S.status), st));
      TraceScope ts(GPT_K_QKV, 1, 0, double(N) * Qc * esz * 2, st);
      GPT_TRY(launch_qkv_post(*c, ws + L.qkv_raw, S.cos_t, S.sin_t, Lb + L.lo.q, Lb + L.lo.k,
                              Lb + L.lo.v, reinterpret_cast<float*>(Lb + L.lo.rq),
                              reinterpret_cast<float*>(Lb + L.lo.rk), st));
    }
    if (has_value_embed(*c, l)) {  // v += 3 sigmoid(h[:, :C] Wg^T) VE[tok], per kv head
      TraceScope ts(GPT_K_OTHER, 1, 0, double(N) * c->n_kv_head * c->head_dim * esz * 3, st);
      GPT_TRY(launch_ve_fwd(*c, Lb + L.lo.h1, S.param(GPT_T_VE_GATE, l), S.param(GPT_T_VE, l), tok,
                            Lb + L.lo.v, st));
    }
    {
      TraceScope ts(GPT_K_ATTN_FWD, 1, attn_f, S.nd() * esz * 4, st);
      GPT_TRY(launch_attn_fwd(*c, Lb + L.lo.q, Lb + L.lo.k, Lb + L.lo.v, Lb + L.lo.o,
                              reinterpret_cast<float*>(Lb + L.lo.lse), S.status, st));
    }
    GPT_TRY(S.projection(gemm_kk(Lb + L.lo.o, d, S.param(GPT_T_WO, l), d, N, d, d,
                                 EPI_RESID_F32, S.x, d, S.status), GPT_T_WO, l));
    GPT_TRY(S.rms_fwd(Lb + L.lo.h2, reinterpret_cast<float*>(Lb + L.lo.r2)));
    GPT_TRY(S.projection(gemm_kk(Lb + L.lo.h2, d, S.param(GPT_T_WUP, l), d, N, F, d,
                                 EPI_RELU2, Lb + L.lo.a, F, S.status), GPT_T_WUP, l));
    GPT_TRY(S.projection(gemm_kk(Lb + L.lo.a, F, S.param(GPT_T_WDOWN, l), F, N, d, F,
                                 EPI_RESID_F32, S.x, d, S.status), GPT_T_WDOWN, l));
    const bool last = l + 1 == c->n_layer;
    if (last && c->backout) {  // x -= backout_lambda x_b before the final norm
      TraceScope ts(GPT_K_OTHER, 1, 0, S.nd() * 12.0, st);
      GPT_TRY(launch_axpy(*c, S.x, S.f(L.xb), static_cast<const char*>(S.param(GPT_T_SCALARS, 0)) + esz,
                          -1.f, st));
    }
    if (!last && c->resid_lambdas) continue;  // the next layer's entry scales x, then normalises it
    void* hn = last ? (void*)(ws + L.hf) : (void*)(S.layer(l + 1) + L.lo.h1);
    float* rn = reinterpret_cast<float*>(last ? ws + L.rf : S.layer(l + 1) + L.lo.r1);
    GPT_TRY(S.rms_fwd(hn, rn));
  }
  // lm_head GEMM with the cross-entropy statistics in its epilogue
  GemmArgs g = gemm_kk(ws + L.hf, d, S.param(GPT_T_LM_HEAD, 0), d, N, V, d, EPI_CE_FWD,
                       nullptr, 0, S.status);
  g.targets = tgt;
  g.part_max = S.f(L.part_max);
  g.part_sum = S.f(L.part_sum);
  g.tgt_logit = S.f(L.tgt_logit);
  g.n_valid = V;
  GPT_TRY(run_gemm(*c, g, st));
  const int tile_n = gemm_ce_tile_n(*c);
  const int n_part = (V + tile_n - 1) / tile_n;
  {
    TraceScope ts(GPT_K_LOSS, 2, 0, double(N) * (n_part * 8.0 + 24), st);
    GPT_TRY(launch_ce_merge(*c, S.f(L.part_max), S.f(L.part_sum), n_part, S.f(L.tgt_logit), tgt,
                            S.f(L.lse_z), S.f(L.tok_loss), S.status, st));
    GPT_TRY(launch_loss_mean(*c, S.f(L.tok_loss), loss, token_loss, S.status, st));
  }
  return GPT_OK;
}

// The backward with a gradient scale and optional per-bucket "gradient
// final" events (gpt_backward_ex in gpt.h).
static int backward_impl(const gpt_config* c, const int32_t* tok, const int32_t* tgt,
                         const void* params, void* workspace, void* grads, int accumulate,
                         float grad_scale, void* const* events, int n_events, void* stream) {
  int rc = check_common(c, tok, tgt, params, workspace);
  if (rc) return rc;
  if (!grads || !aligned(grads, 256) || (accumulate != 0 && accumulate != 1)) return GPT_EINVAL;
  if (!std::isfinite(grad_scale) || !(grad_scale > 0.f)) return GPT_EINVAL;
  if (events && n_events != c->n_layer + 2) return GPT_EINVAL;
  for (int i = 0; events && i < n_events; ++i)
    if (!events[i]) return GPT_EINVAL;
  auto mark = [&](int i) -> int {  // the gradients of bucket i are final on `stream`
    return events ? int(cudaEventRecord(static_cast<cudaEvent_t>(events[i]), (cudaStream_t)stream))
                  : 0;
  };
  Step S(c, workspace, params, stream);
  const Layout& L = S.L;
  const int N = S.N, d = S.d, F = S.F, V = S.V, esz = S.esz;
  char* ws = S.ws;
  cudaStream_t st = S.st;
  int32_t* status = S.status;
  char* gr = static_cast<char*>(grads);
  auto grad = [&](int t, int l) -> void* {
    int64_t off, r, cc;
    gpt_param_offset(c, t, l, &off, &r, &cc);
    return gr + off * esz;
  };

  {
    TraceScope ts(GPT_K_SORT, 8, 0, double(N) * 12 + double(V) * 16, st);
    GPT_TRY(launch_sort_tokens(*c, L, tok, ws, st));
  }
  if (c->fp8 && c->n_layer > 0) GPT_TRY(S.quant_weights_t());
  // logits gradient G = (softmax(z) - onehot(target)) / N, recomputed from the saved lse
  GemmArgs g = gemm_kk(ws + L.hf, d, S.param(GPT_T_LM_HEAD, 0), d, N, int(L.vpad), d,
                       EPI_CE_BWD, ws + L.G, L.vpad, status);
  g.targets = tgt;
  g.lse = S.f(L.lse_z);
  g.inv_n = grad_scale / float(N);
  g.n_valid = V;
  GPT_TRY(run_gemm(*c, g, st));
  // dhf = G Wlm ; dWlm = G^T hf
  g = gemm_kk(ws + L.G, L.vpad, S.param(GPT_T_LM_HEAD, 0), d, N, d, V, EPI_STORE, ws + L.dh, d,
              status);
  g.b_mn_major = true;
  GPT_TRY(run_gemm(*c, g, st));
  g = gemm_kk(ws + L.G, L.vpad, ws + L.hf, d, V, d, N, EPI_STORE, grad(GPT_T_LM_HEAD, 0), d,
              status);
  g.a_mn_major = true; g.b_mn_major = true; g.beta = accumulate;
  GPT_TRY(run_gemm(*c, g, st));
  GPT_TRY(cuda_rc(cudaError_t(mark(0))));
  GPT_TRY(S.rms_bwd(ws + L.dh, ws + L.hf, S.f(L.rf), 0));
  const uint64_t nd4 = uint64_t(N) * d * 4;
  char* gvar_scalars = (c->smear || c->backout) ? static_cast<char*>(grad(GPT_T_SCALARS, 0)) : nullptr;
  if (c->backout) {  // x_out = x_L - beta x_b: d beta = -sum(dx_out x_b); keep dx_out
    TraceScope ts(GPT_K_OTHER, 3, 0, S.nd() * 16.0, st);
    GPT_TRY(cuda_rc(cudaMemcpyAsync(ws + L.dxf, S.x, nd4, cudaMemcpyDeviceToDevice, st)));
    GPT_TRY(launch_dot(*c, S.f(L.dxf), S.f(L.xb), -1.f, S.f(L.vred), gvar_scalars + esz, accumulate, st));
  }
  if (c->resid_lambdas) GPT_TRY(cuda_rc(cudaMemsetAsync(ws + L.dx0, 0, nd4, st)));

  const double attn_b = 8.0 * attn_pairs(*c) * c->head_dim;  // dV, dP, dQ, dK, causal half
  // bf16 steps fold the MLP norm's backward into the two MLP data-gradient
  // GEMMs.  With h = h2 the norm's output, u = h Wup^T, a = relu(u)^2 and
  // dh = du Wup, the row sum that the RMSNorm backward needs is
  //   sum_j dh_j h_j = sum_f du_f u_f = 2 sum_f da_f a_f
  // (du = da * 2 relu(u) is 0 where u <= 0, and relu(u) u = a elsewhere):
  // the down-projection dgrad's epilogue has da and a in hand and writes
  // per-row partials of it; the up-projection dgrad's epilogue sums them and
  // applies dx += r (dh - h s), s = (2/d) sum, writing the bf16 copy of dx.
  const bool fold = c->dtype == GPT_BF16 && !c->fp8;
  const int n_np = (F + gemm_ce_tile_n(*c) - 1) / gemm_ce_tile_n(*c);
  for (int l = c->n_layer - 1; l >= 0; --l) {
    char* Lb = S.layer(l);
    // MLP down: da = dx Wdown, du = da * 2 relu(u) (from the stored a = relu(u)^2)
    g = gemm_kk(ws + L.dxs, d, S.param(GPT_T_WDOWN, l), F, N, F, d, EPI_DRELU2, ws + L.du, F,
                status);
    g.b_mn_major = true; g.aux = Lb + L.lo.a;
    if (fold) { g.norm_part_out = S.f(L.npart); g.n_npart = n_np; }
    GPT_TRY(S.dgrad(g, GPT_T_WDOWN, l));
    g = gemm_kk(ws + L.dxs, d, Lb + L.lo.a, F, d, F, N, EPI_STORE, grad(GPT_T_WDOWN, l), F,
                status);
    g.a_mn_major = true; g.b_mn_major = true; g.beta = accumulate;
    GPT_TRY(run_gemm(*c, with_splitk(g, L, ws), st));
    // MLP up (with the norm's backward when folded)
    float* r2 = reinterpret_cast<float*>(Lb + L.lo.r2);
    g = gemm_kk(ws + L.du, F, S.param(GPT_T_WUP, l), d, N, d, F, fold ? EPI_NORM_BWD : EPI_STORE,
                fold ? static_cast<void*>(S.x) : ws + L.dh, d, status);
    g.b_mn_major = true;
    if (fold) {
      g.aux = Lb + L.lo.h2; g.out2 = ws + L.dxs; g.norm_part = S.f(L.npart); g.norm_r = r2;
      g.n_npart = n_np; g.norm_scale = 2.f / float(d);
    }
    GPT_TRY(S.dgrad(g, GPT_T_WUP, l));
    g = gemm_kk(ws + L.du, F, Lb + L.lo.h2, d, F, d, N, EPI_STORE, grad(GPT_T_WUP, l), d, status);
    g.a_mn_major = true; g.b_mn_major = true; g.beta = accumulate;
    GPT_TRY(run_gemm(*c, with_splitk(g, L, ws), st));
    if (!fold) GPT_TRY(S.rms_bwd(ws + L.dh, Lb + L.lo.h2, r2, 1));
    // attention out-projection
    g = gemm_kk(ws + L.dxs, d, S.param(GPT_T_WO, l), d, N, d, d, EPI_STORE, ws + L.dO, d, status);
    g.b_mn_major = true;
    GPT_TRY(S.dgrad(g, GPT_T_WO, l));
    g = gemm_kk(ws + L.dxs, d, Lb + L.lo.o, d, d, d, N, EPI_STORE, grad(GPT_T_WO, l), d, status);
    g.a_mn_major = true; g.b_mn_major = true; g.beta = accumulate;
    GPT_TRY(run_gemm(*c, with_splitk(g, L, ws), st));
    // attention, then QK-norm and RoPE backward, into dqkv [N, Q] (Q = qkv columns);
    // folded: the attention kernels also write the input norm's row partials
    // (sum_j dh_j h_j = sum_c dqkv_c qkv_c with qkv = h Wqkv^T the raw
    // projection, per head), and the QKV dgrad's epilogue applies the norm's
    // backward.  Not with a value embedding in this layer: its v is not the
    // projection's, and its gate adds to dh after the GEMM.
    const bool ve = has_value_embed(*c, l);
    const bool fold_attn = fold && !ve;
    {
      TraceScope ts(GPT_K_ATTN_BWD, 2, attn_b, S.nd() * esz * 8, st);
      GPT_TRY(launch_attn_bwd(*c, Lb + L.lo.q, Lb + L.lo.k, Lb + L.lo.v, Lb + L.lo.o, ws + L.dO,
                              reinterpret_cast<float*>(Lb + L.lo.lse),
                              reinterpret_cast<float*>(Lb + L.lo.rq),
                              reinterpret_cast<float*>(Lb + L.lo.rk), S.cos_t, S.sin_t,
                              S.f(L.Dattn), ws + L.dqkv, fold_attn ? S.f(L.npart) : nullptr,
                              S.status, st));
    }
    if (ve) {  // the value embedding's table and gate gradients from dv
      TraceScope ts(GPT_K_OTHER, 2, 0, double(N) * c->n_kv_head * c->head_dim * (esz * 2 + 4), st);
      GPT_TRY(launch_ve_bwd(*c, ws + L.dqkv, Lb + L.lo.h1, S.param(GPT_T_VE_GATE, l), S.param(GPT_T_VE, l),
                            tok, S.f(L.ve_rows), S.f(L.ve_dgz), grad(GPT_T_VE_GATE, l), accumulate, st));
      gpt_config cv = *c;
      cv.d_model = c->n_kv_head * c->head_dim;
      TraceScope ts2(GPT_K_SCATTER, 5, 0, double(N) * cv.d_model * 4 + double(V) * cv.d_model * esz, st);
      GPT_TRY(launch_embed_scatter(cv, L, S.f(L.ve_rows), ws, grad(GPT_T_VE, l), accumulate, st));
    }
    const int Qc = int(qkv_cols(*c));
    float* r1 = reinterpret_cast<float*>(Lb + L.lo.r1);
    g = gemm_kk(ws + L.dqkv, Qc, S.param(GPT_T_WQKV, l), d, N, d, Qc,
                fold_attn ? EPI_NORM_BWD : EPI_STORE, fold_attn ? static_cast<void*>(S.x) : ws + L.dh,
                d, status);
    g.b_mn_major = true;
    if (fold_attn) {
      g.aux = Lb + L.lo.h1; g.out2 = ws + L.dxs; g.norm_part = S.f(L.npart); g.norm_r = r1;
      g.n_npart = c->n_head + 2 * c->n_kv_head; g.norm_scale = 1.f / float(d);
    }
    GPT_TRY(S.dgrad(g, GPT_T_WQKV, l));
    if (ve) {  // the gate's input h[:, :C]
      TraceScope ts(GPT_K_OTHER, 1, 0, double(N) * c->ve_gate_channels * esz * 2, st);
      GPT_TRY(launch_ve_dh(*c, ws + L.dh, S.f(L.ve_dgz), S.param(GPT_T_VE_GATE, l), st));
    }
    g = gemm_kk(ws + L.dqkv, Qc, Lb + L.lo.h1, d, Qc, d, N, EPI_STORE,
                grad(GPT_T_WQKV, l), d, status);
    g.a_mn_major = true; g.b_mn_major = true; g.beta = accumulate;
    GPT_TRY(run_gemm(*c, with_splitk(g, L, ws), st));
    GPT_TRY(cuda_rc(cudaError_t(mark(1 + l))));  // every weight gradient of layer l is final
    if (!fold_attn) GPT_TRY(S.rms_bwd(ws + L.dh, Lb + L.lo.h1, r1, 1));
    const bool bo = c->backout && l == backout_layer(*c);
    if (bo || c->resid_lambdas) {  // the layer's entry: backout point, residual scaling
      TraceScope ts(GPT_K_OTHER, c->resid_lambdas ? 2 : 1, 0, S.nd() * (c->resid_lambdas ? 26.0 : 14.0), st);
      const char* lam =
          c->resid_lambdas ? static_cast<const char*>(S.param(GPT_T_LAMBDAS, 0)) + int64_t(l) * 2 * esz : nullptr;
      char* dlam = c->resid_lambdas ? static_cast<char*>(grad(GPT_T_LAMBDAS, 0)) + int64_t(l) * 2 * esz : nullptr;
      GPT_TRY(launch_resid_bwd(*c, S.x, ws + L.dxs, bo ? S.f(L.dxf) : nullptr,
                               bo ? S.param(GPT_T_SCALARS, 0) : nullptr,
                               c->resid_lambdas ? S.f(L.xprev + uint64_t(l) * nd4) : nullptr,
                               c->resid_lambdas ? S.f(L.x0) : nullptr, c->resid_lambdas ? S.f(L.dx0) : nullptr,
                               lam, S.f(L.vred), dlam, accumulate, st));
    }
  }
  if (c->resid_lambdas) {  // x0 is the stream entering layer 0
    TraceScope ts(GPT_K_OTHER, 1, 0, S.nd() * 12.0, st);
    GPT_TRY(launch_axpy(*c, S.x, S.f(L.dx0), nullptr, 1.f, st));
  }
  if (c->smear) {  // back through x = e + s sigmoid(e[:24] . w) e_prev, into L.emb
    TraceScope ts(GPT_K_OTHER, 4, 0, S.nd() * 16.0, st);
    GPT_TRY(launch_smear_bwd(*c, S.x, S.f(L.emb), S.f(L.sm_sg), S.f(L.sm_dg), S.f(L.sm_du),
                             S.param(GPT_T_SMEAR_GATE, 0), S.param(GPT_T_SCALARS, 0),
                             grad(GPT_T_SMEAR_GATE, 0), gvar_scalars, accumulate, st));
  }
  {
    TraceScope ts(GPT_K_SCATTER, 6, 0, S.nd() * 4 + double(V) * d * esz, st);
    GPT_TRY(launch_embed_scatter(*c, L, c->smear ? S.f(L.emb) : S.x, ws, grad(GPT_T_WTE, 0), accumulate, st));
  }
  GPT_TRY(cuda_rc(cudaError_t(mark(c->n_layer + 1))));
  return GPT_OK;
}

int gpt_backward(const gpt_config* c, const int32_t* tok, const int32_t* tgt,
                 const void* params, void* workspace, void* grads, int accumulate,
                 void* stream) {
  return backward_impl(c, tok, tgt, params, workspace, grads, accumulate, 1.0f, nullptr, 0, stream);
}

int gpt_backward_ex(const gpt_config* c, const int32_t* tok, const int32_t* tgt,
                    const void* params, void* workspace, void* grads, int accumulate,
                    float grad_scale, void* const* grad_ready_events, int n_events, void* stream) {
  return backward_impl(c, tok, tgt, params, workspace, grads, accumulate, grad_scale,
                       grad_ready_events, n_events, stream);
}

int gpt_train_step_host(const gpt_config* c, const int32_t* host_tokens,
                        const int32_t* host_targets, const void* params, void* workspace,
                        void* grads, int accumulate, float* host_loss, void* stream) {
  if (!c || !host_tokens || !host_targets || !workspace || !host_loss) return GPT_EINVAL;
  if (!aligned(workspace, 256)) return GPT_EINVAL;
  Layout L;
  make_layout(*c, &L);
  char* ws = static_cast<char*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* dtok = reinterpret_cast<int32_t*>(ws + L.tok_stage);
  int32_t* dtgt = reinterpret_cast<int32_t*>(ws + L.tgt_stage);
  float* dloss = reinterpret_cast<float*>(ws + L.loss_acc);
  const size_t nb = size_t(L.N) * 4;
  if (cudaMemcpyAsync(dtok, host_tokens, nb, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return GPT_ECUDA;
  if (cudaMemcpyAsync(dtgt, host_targets, nb, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return GPT_ECUDA;
  int rc = gpt_forward_loss(c, dtok, dtgt, params, workspace, dloss, nullptr, stream);
  if (rc) return rc;
  rc = gpt_backward(c, dtok, dtgt, params, workspace, grads, accumulate, stream);
  if (rc) return rc;
  if (cudaMemcpyAsync(host_loss, dloss, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return GPT_ECUDA;
  return GPT_OK;
}

int gpt_status(const void* workspace, void* stream) {
  if (!workspace) return GPT_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return GPT_ECUDA;
  gpt_device_status s;
  if (cudaMemcpy(&s, workspace, sizeof(s), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GPT_ECUDA;
  return s.code;
}

int gpt_wait_expiry_check(void* workspace, int64_t limit_ns, void* stream) {
  if (!workspace || !aligned(workspace, 256)) return GPT_EINVAL;
  if (limit_ns < 1000 || limit_ns > 10000000000ll) return GPT_EINVAL;
  return launch_wait_expiry(static_cast<int32_t*>(workspace), uint64_t(limit_ns), stream) ? GPT_ECUDA
                                                                                         : GPT_OK;
}

// ---------------------------------------------------------------------------
// optimizer step ("ChatGPT'nizi 50 Dolara Nasil Egitirsiniz?", section "2. Muon
// Optimize Edici (nanochat/optim.py)"): AdamW for wte and lm_head, Muon for
// the block matrices
// ---------------------------------------------------------------------------
int gpt_optim_defaults(gpt_optim* o) {
  if (!o) return GPT_EINVAL;
  *o = gpt_optim{};
  // library defaults (the pages give no values): Adam's published
  // suggestions, a common Muon setting, the two printed coefficient triples
  o->adam_lr = 1e-3f;
  o->adam_beta1 = 0.9f;
  o->adam_beta2 = 0.999f;
  o->adam_eps = 1e-8f;
  o->adam_weight_decay = 0.f;
  o->muon_lr = 0.02f;
  o->muon_momentum = 0.95f;
  o->muon_nesterov = 1;
  o->ns_steps = 2;
  const float printed[2][3] = {{8.156f, -22.483f, 15.879f}, {4.043f, -2.809f, 0.500f}};
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 3; ++j) o->ns_coeffs[i][j] = printed[i][j];
  o->step = 1;
  o->normuon = 0;
  o->normuon_beta2 = 0.95f;
  return GPT_OK;
}

static int check_optim_cfg(const gpt_config* c) {
  if (!c) return GPT_EINVAL;
  gpt_config chk = *c;
  int rc = gpt_config_init(&chk);
  if (rc != GPT_OK) return rc;
  if (chk.param_bytes != c->param_bytes || chk.workspace_bytes != c->workspace_bytes)
    return GPT_EINVAL;
  if (c->dtype != GPT_BF16) return GPT_EUNSUPPORTED;
  return GPT_OK;
}

int gpt_optim_state_bytes(const gpt_config* c, size_t* bytes) {
  if (!bytes) return GPT_EINVAL;
  const int rc = check_optim_cfg(c);
  if (rc != GPT_OK) return rc;
  *bytes = size_t(3) * (c->param_bytes / 2) * 4;
  return GPT_OK;
}

int gpt_optim_init(const gpt_config* c, const void* params, void* state, void* stream) {
  const int rc = check_optim_cfg(c);
  if (rc != GPT_OK) return rc;
  if (!params || !state || !aligned(params, 256) || !aligned(state, 256)) return GPT_EINVAL;
  const int64_t pe = int64_t(c->param_bytes / 2);
  float* w = static_cast<float*>(state);
  return launch_optim_init(params, w, w + pe, w + 2 * pe, pe, stream) ? GPT_ECUDA : GPT_OK;
}

int gpt_optim_step(const gpt_config* c, const gpt_optim* o, void* params, const void* grads,
                   void* state, void* workspace, void* stream) {
  int rc = check_optim_cfg(c);
  if (rc != GPT_OK) return rc;
  if (!o || !params || !grads || !state || !workspace) return GPT_EINVAL;
  if (!aligned(params, 256) || !aligned(grads, 256) || !aligned(state, 256) || !aligned(workspace, 256))
    return GPT_EINVAL;
  if (o->ns_steps < 0 || o->ns_steps > 8 || o->step < 1) return GPT_EINVAL;
  const float hp[] = {o->adam_lr, o->adam_beta1, o->adam_beta2, o->adam_eps, o->adam_weight_decay,
                      o->muon_lr, o->muon_momentum};
  for (float x : hp)
    if (!std::isfinite(x)) return GPT_EINVAL;
  for (int i = 0; i < o->ns_steps; ++i)
    for (int j = 0; j < 3; ++j)
      if (!std::isfinite(o->ns_coeffs[i][j])) return GPT_EINVAL;
  if (!(o->adam_beta1 >= 0.f && o->adam_beta1 < 1.f && o->adam_beta2 >= 0.f && o->adam_beta2 < 1.f))
    return GPT_EINVAL;
  if (o->muon_nesterov != 0 && o->muon_nesterov != 1) return GPT_EINVAL;
  if (o->normuon != 0 && o->normuon != 1) return GPT_EINVAL;
  if (o->normuon && !(o->normuon_beta2 >= 0.f && o->normuon_beta2 < 1.f)) return GPT_EINVAL;

  cudaStream_t st = (cudaStream_t)stream;
  Layout L;
  make_layout(*c, &L);
  char* ws = static_cast<char*>(workspace);
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  const int64_t pe = int64_t(c->param_bytes / 2);
  float* W = static_cast<float*>(state);
  float* M = W + pe;
  float* Vv = M + pe;
  auto* P = static_cast<__nv_bfloat16*>(params);
  auto* G = static_cast<const __nv_bfloat16*>(grads);

  // AdamW: the embedding and lm_head
  const double t = double(o->step);
  const float bc1 = float(1.0 - std::pow(double(o->adam_beta1), t));
  const float bc2 = float(1.0 - std::pow(double(o->adam_beta2), t));
  // AdamW: the embedding, lm_head and every block-variant parameter (value
  // embeddings and their gates, scales), each over its aligned span (the
  // padding's gradient and state are zero and stay zero)
  std::vector<std::pair<int, int>> adam = {{GPT_T_WTE, 0}, {GPT_T_LM_HEAD, 0}};
  for (int l = 0; l < c->n_layer; ++l)
    if (has_value_embed(*c, l)) {
      adam.push_back({GPT_T_VE, l});
      adam.push_back({GPT_T_VE_GATE, l});
    }
  if (c->resid_lambdas) adam.push_back({GPT_T_LAMBDAS, 0});
  if (c->smear) adam.push_back({GPT_T_SMEAR_GATE, 0});
  if (c->smear || c->backout) adam.push_back({GPT_T_SCALARS, 0});
  for (auto [tensor, layer] : adam) {
    int64_t off, r, cc;
    gpt_param_offset(c, tensor, layer, &off, &r, &cc);
    const int64_t n = param_elems_aligned(r * cc);
    TraceScope ts(GPT_K_OTHER, 1, 0, double(n) * 30.0, st);
    GPT_TRY(launch_adamw(P + off, G + off, W + off, M + off, Vv + off, n, o->adam_lr, o->adam_beta1,
                         o->adam_beta2, o->adam_eps, o->adam_weight_decay, bc1, bc2, st));
  }
  // Muon: every block matrix.  One kind of matrix (same shape in every layer)
  // is orthogonalised for all layers together: the momentum pass writes each
  // layer's X into a stacked [n_layer, rows, cols] buffer and every
  // Newton-Schulz product is one batched GEMM over the layers.
  char* x0 = ws + L.opt_x0;
  char* x1 = ws + L.opt_x1;
  char* A = ws + L.opt_a;
  char* Bm = ws + L.opt_b;
  float* part = reinterpret_cast<float*>(ws + L.opt_part);
  const int nl = c->n_layer;
  // one batched product; per-layer launches when a K block would straddle two
  // layers' rows (K not a multiple of the 64-wide K block)
  auto batched = [&](GemmArgs g, int64_t a_bs, int64_t b_bs, int64_t o_bs, bool split) -> int {
    if (g.K % 64 == 0) {
      g.batch = nl;
      g.a_bstride = a_bs;
      g.b_bstride = b_bs;
      g.o_bstride = o_bs;
      return run_gemm(*c, g, st);
    }
    for (int l = 0; l < nl; ++l) {
      GemmArgs gl = g;
      gl.A = static_cast<const __nv_bfloat16*>(g.A) + l * a_bs * g.lda;
      gl.B = static_cast<const __nv_bfloat16*>(g.B) + l * b_bs * g.ldb;
      gl.out = static_cast<__nv_bfloat16*>(g.out) + l * o_bs * g.ldo;
      if (g.aux) gl.aux = static_cast<const __nv_bfloat16*>(g.aux) + l * o_bs * g.ldo;
      const int rc = run_gemm(*c, split ? with_splitk(gl, L, ws) : gl, st);
      if (rc) return rc;
    }
    return 0;
  };
  for (int tensor : {GPT_T_WQKV, GPT_T_WO, GPT_T_WUP, GPT_T_WDOWN}) {
    int64_t off0, r, cc;
    gpt_param_offset(c, tensor, 0, &off0, &r, &cc);
    const int64_t n = r * cc;
    for (int l = 0; l < nl; ++l) {
      int64_t off, rr, rc2;
      gpt_param_offset(c, tensor, l, &off, &rr, &rc2);
      TraceScope ts(GPT_K_OTHER, 3, 0, double(n) * 16.0, st);
      GPT_TRY(launch_muon_prepare(G + off, M + off, n, o->muon_momentum, o->muon_nesterov, part,
                                  x0 + l * n * 2, st));
    }
    // Newton-Schulz on each X [r, cc]; the Gram matrix is gd x gd over the smaller side
    const bool tall = r >= cc;
    const int gd = int(tall ? cc : r);
    char* X = x0;
    char* Xn = x1;
    for (int i = 0; i < o->ns_steps; ++i) {
      const float a = o->ns_coeffs[i][0], b = o->ns_coeffs[i][1], cf = o->ns_coeffs[i][2];
      // A = X^T X (tall: both operands are X read MN-major) or X X^T (wide)
      GemmArgs g1 = gemm_kk(X, cc, X, cc, gd, gd, int(tall ? r : cc), EPI_STORE, A, gd, status);
      g1.a_mn_major = tall;
      g1.b_mn_major = tall;
      GPT_TRY(batched(g1, r, r, gd, true));
      // B = c A A + b A
      GemmArgs g2 = gemm_kk(A, gd, A, gd, gd, gd, gd, EPI_AXPBY, Bm, gd, status);
      g2.b_mn_major = true;
      g2.aux = A;
      g2.alpha = cf;
      g2.beta_aux = b;
      GPT_TRY(batched(g2, gd, gd, gd, false));
      // X' = X B + a X (tall) or B X + a X (wide)
      GemmArgs g3 = tall ? gemm_kk(X, cc, Bm, gd, int(r), int(cc), gd, EPI_AXPBY, Xn, cc, status)
                         : gemm_kk(Bm, gd, X, cc, int(r), int(cc), gd, EPI_AXPBY, Xn, cc, status);
      g3.b_mn_major = true;
      g3.aux = X;
      g3.alpha = 1.f;
      g3.beta_aux = a;
      GPT_TRY(batched(g3, tall ? r : gd, tall ? gd : r, r, false));
      std::swap(X, Xn);
    }
    const float step = o->muon_lr * std::sqrt(std::max(1.f, float(r) / float(cc)));
    float* vmean = reinterpret_cast<float*>(ws + L.opt_rows);
    float* factor = vmean + std::max(std::max(qkv_cols(*c), int64_t(c->d_ff)), int64_t(c->d_model));
    for (int l = 0; l < nl; ++l) {
      int64_t off, rr, rc2;
      gpt_param_offset(c, tensor, l, &off, &rr, &rc2);
      if (o->normuon) {
        // NorMuon: the per-row state lives in this matrix's (otherwise unused)
        // second-moment slots of the state buffer
        TraceScope ts(GPT_K_OTHER, 3, 0, double(n) * 2.0 + double(r) * 16.0, st);
        GPT_TRY(launch_normuon(X + l * n * 2, Vv + off, int(r), int(cc), o->normuon_beta2, vmean, factor, st));
        TraceScope ts2(GPT_K_OTHER, 1, 0, double(n) * 12.0, st);
        GPT_TRY(launch_muon_apply_rows(X + l * n * 2, W + off, P + off, int(r), int(cc), step, factor, st));
      } else {
        TraceScope ts(GPT_K_OTHER, 1, 0, double(n) * 12.0, st);
        GPT_TRY(launch_muon_apply(X + l * n * 2, W + off, P + off, n, step, st));
      }
    }
  }
  return GPT_OK;
}

}  // extern "C"
