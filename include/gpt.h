/*
 * gpt.h -- C ABI of libgpt: one forward + backward training step of a
 * pre-norm decoder-only GPT on one NVIDIA B200 (sm_100a).
 *
 * The model is the one sketched in "ChatGPT'nizi 50 Dolara Nasil
 * Egitirsiniz?" (dev.to), section "1. GPT Modeli (nanochat/gpt.py)": rotary
 * position embeddings, QK normalisation, untied token embedding and lm_head,
 * ReLU^2 MLP, causal attention (section "5. Flash Dikkat Mekanizmasi
 * Birlesimi", causal=True, optionally with a sliding window), optionally
 * grouped-query attention (the model list), bias-free linear layers (section "3. Hassasiyet
 * Yonetimi", F.linear(x, W) with W stored [out, in]).  Width, heads and MLP
 * size follow the depth dial of section "Felsefe: Her Seyi Kontrol Eden Tek
 * Bir Kadran" (d_model = 64 * depth, head_dim 128, d_ff = 4 * d_model).
 *
 * Step, per sequence of T tokens (all norms parameter-free RMSNorm,
 * y = x / sqrt(mean(x^2) + eps)):
 *   x = wte[tokens]
 *   per layer:  h = rms(x); [q|k|v] = h Wqkv^T; q,k <- rms_head(RoPE(q,k))
 *               x += causal_softmax(q k^T / sqrt(hd)) v  Wo^T
 *               (k, v: n_kv_head heads, each shared by n_head/n_kv_head
 *               consecutive query heads; keys restricted to the last
 *               attn_window positions when that is set)
 *               h = rms(x); x += relu(h Wup^T)^2 Wdown^T
 *   z = rms(x) Wlm^T;  loss = mean_t (logsumexp(z_t) - z_t[target_t])
 * and the exact gradient of that loss w.r.t. every parameter.
 *
 * Conventions for every call below:
 *  - All device buffers are owned by the caller; the library allocates no
 *    device memory and keeps no global mutable state (except the scratch
 *    array of gpt_embedding_grad_noalloc, described there).  Pointers marked
 *    "device" must be device memory of the current CUDA device.
 *  - Device pointers must be 16-byte aligned (TMA); params/grads/workspace
 *    256-byte aligned.  A violation returns GPT_EINVAL before any launch.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t, NULL = the
 *    legacy default stream).  Results are deterministic: bit-identical
 *    across runs for identical inputs (no floating-point atomics).
 *  - Return value 0 on success, a negative GPT_E* code otherwise.  Errors
 *    found on the device (bad token ids, an expired bounded wait, a
 *    non-finite loss) are recorded in the workspace and read by gpt_status().
 */
#ifndef GPT_B200_H
#define GPT_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- error codes ------------------------------------------------------ */
#define GPT_OK 0
#define GPT_EINVAL (-1)       /* null / misaligned pointer, inconsistent config */
#define GPT_EUNSUPPORTED (-2) /* shape or dtype outside what the kernels cover  */
#define GPT_ECUDA (-3)        /* a CUDA runtime / driver call failed            */
#define GPT_EDATA (-4)        /* a token or target id outside [0, vocab)        */
#define GPT_ETIMEOUT (-5)     /* a bounded device-side wait expired             */
#define GPT_ENONFINITE (-6)   /* the loss came out NaN or Inf                   */

/* ---- storage types ---------------------------------------------------- */
#define GPT_BF16 0 /* bf16 params/activations/grads, fp32 accumulate (tensor cores) */
#define GPT_F32 1  /* fp32 everywhere (small models; SIMT kernels)                  */

/* ---- parameter tensors (for gpt_param_offset) -------------------------- */
#define GPT_T_WTE 0     /* [vocab, d_model]          token embedding          */
#define GPT_T_WQKV 1    /* [d_model + 2*n_kv_head*head_dim, d_model] (3*d_model
                           without GQA): the n_head q heads' rows, then the
                           n_kv_head k heads', then the v heads'; inside each
                           block head h owns rows h*hd..h*hd+hd-1             */
#define GPT_T_WO 2      /* [d_model, d_model]        attention out-projection */
#define GPT_T_WUP 3     /* [d_ff, d_model]           MLP up                   */
#define GPT_T_WDOWN 4   /* [d_model, d_ff]           MLP down                 */
#define GPT_T_LM_HEAD 5 /* [vocab, d_model]          untied output head       */
/* Block-variant parameters (present only when their config field is on; they
 * follow lm_head in the flat buffer, in this order): */
#define GPT_T_VE 6         /* [vocab, n_kv_head*head_dim] value embedding of layer l
                              (layers l with l % ve_every == ve_every - 1)       */
#define GPT_T_VE_GATE 7    /* [n_kv_head, ve_gate_channels] its gate             */
#define GPT_T_LAMBDAS 8    /* [n_layer, 2]: (resid, x0) scale of each layer      */
#define GPT_T_SMEAR_GATE 9 /* [1, 24]: smear gate on the embedding's 24 channels */
#define GPT_T_SCALARS 10   /* [1, 2]: (smear scale, backout scale)               */

/* ---- workspace regions (for gpt_workspace_region, diagnostics/tests) ---- */
#define GPT_W_STATUS 0     /* gpt_device_status struct                                 */
#define GPT_W_RESID 1      /* fp32 [N, d]: residual stream.  After gpt_forward_loss it */
                           /*   holds the last layer's output (x0 = wte[tokens], exact, */
                           /*   when n_layer == 0); after gpt_backward, d loss / d x0   */
#define GPT_W_LSE 2        /* fp32 [N]: logsumexp of each position's logits           */
#define GPT_W_SORT_PERM 3  /* int32 [N]: positions stably sorted by token id          */
#define GPT_W_SORT_OFFS 4  /* int32 [vocab+1]: segment starts in SORT_PERM            */
#define GPT_W_ATTN_LSE 5   /* fp32 [B, H, T] of layer `layer`: row logsumexp of the    */
                           /*   scaled attention scores                                */

/* Device-side status, at the start of the workspace. */
typedef struct gpt_device_status {
  int32_t code;      /* 0 or the first GPT_E* recorded              */
  int32_t where;     /* kernel id that recorded it (diagnostic)      */
  int64_t index;     /* offending token position / wait site         */
  int32_t reserved[12];
} gpt_device_status;

typedef struct gpt_config {
  /* model and batch shape (set by the caller) */
  int32_t n_layer;  /* >= 0                                             */
  int32_t d_model;  /* = n_head * head_dim                               */
  int32_t n_head;
  int32_t head_dim; /* bf16: 64 or 128; f32: even, <= 128               */
  int32_t d_ff;     /* bf16: multiple of 64; f32: any >= 1              */
  int32_t vocab;    /* >= 2                                              */
  int32_t seq_len;  /* T >= 1                                            */
  int32_t batch;    /* B >= 1                                            */
  int32_t dtype;    /* GPT_BF16 or GPT_F32                               */
  int32_t qk_norm;  /* 1: RMSNorm q and k per head after RoPE (default)  */
  int32_t n_kv_head;   /* key/value heads (grouped-query attention): query
                          head h reads key/value head h / (n_head/n_kv_head);
                          divides n_head; 0 = n_head (set by gpt_config_init) */
  int32_t attn_window; /* sliding window: query i attends to keys i-W < j <= i
                          in every layer; 0 = the full causal window          */
  int32_t fp8;         /* 1: the forward block projections (Wqkv, Wo, Wup,
                          Wdown) multiply e4m3 operands -- activations scaled
                          per row, weights per tensor, by powers of two -- and
                          the backward stays bf16 (straight-through); bf16
                          configs only                                        */
  /* Block variants ("ChatGPT'nizi 50 Dolara Nasil Egitirsiniz?", section
   * "1. GPT Modeli": the value-embedding and efficiency-trick listings); each
   * one's parameters are inputs like every other weight (GPT_T_VE ..
   * GPT_T_SCALARS), so their initial values are the caller's: */
  int32_t ve_every;    /* k >= 1: layers l with l % k == k - 1 add a gated value
                          embedding to v, v += 3 sigmoid(h[:, :C] Wg^T) VE[token]
                          per key/value head (h: the block's normalised input);
                          0 = none                                             */
  int32_t ve_gate_channels; /* C, 1 .. d_model; 0 = 32 (capped at d_model)     */
  int32_t resid_lambdas;    /* 1: x = lam[l,0] x + lam[l,1] x0 on entering layer l
                               (x0: the stream entering layer 0)               */
  int32_t smear;       /* 1: after the gather, x_t = e_t + s sigmoid(e_t[:24] . w)
                          e_{t-1} (s = scalars[0]; nothing at a sequence start);
                          d_model >= 24                                        */
  int32_t backout;     /* 1: x = x - scalars[1] x_b before the final norm, x_b the
                          stream entering layer n_layer / 2                    */
  float rope_base;  /* 10000 by default                                  */
  float norm_eps;   /* 1e-6 by default                                   */
  /* derived by gpt_config_init */
  int64_t n_params;        /* parameter count                               */
  uint64_t param_bytes;    /* bytes of the flat parameter (and grad) buffer */
  uint64_t workspace_bytes;/* bytes of the workspace                        */
} gpt_config;

/* Validate `cfg` and fill its derived fields.  Host only, no CUDA call.
 * Zero-valued rope_base / norm_eps / n_kv_head are replaced by the defaults.
 * GPT_EINVAL for a NULL or inconsistent config (d_model != n_head*head_dim,
 * non-positive sizes, n_kv_head not dividing n_head, attn_window < 0),
 * GPT_EUNSUPPORTED for shapes the kernels do not cover
 * (bf16: d_model % 64, d_ff % 64, head_dim not 64/128; f32: odd head_dim or
 * head_dim > 128). */
int gpt_config_init(gpt_config* cfg);

/* The depth dial: d_model = 64*depth, head_dim = 128, n_head = depth/2,
 * d_ff = 4*d_model, n_layer = depth, bf16, qk_norm on, defaults for eps and
 * RoPE base; then gpt_config_init.  depth must be even and >= 2. */
int gpt_config_from_depth(gpt_config* cfg, int depth, int seq_len, int batch, int vocab);

/* Element offset and [rows, cols] of one parameter tensor inside the flat
 * parameter buffer (the grad buffer has the same layout).  Tensors are
 * row-major [out, in].  `layer` is ignored for GPT_T_WTE / GPT_T_LM_HEAD.
 * Order in the buffer: wte, then per layer wqkv, wo, wup, wdown, then lm_head;
 * every tensor starts on a 128-element boundary. */
int gpt_param_offset(const gpt_config* cfg, int tensor, int layer, int64_t* elem_offset,
                     int64_t* rows, int64_t* cols);

/* Byte offset and size of a workspace region (GPT_W_*); `layer` is used by
 * per-layer regions only. */
int gpt_workspace_region(const gpt_config* cfg, int region, int layer, uint64_t* byte_offset,
                         uint64_t* bytes);

/* Forward pass and loss.
 *   tokens, targets: device int32 [batch, seq_len], row-major.
 *   params:          device, flat buffer of cfg->param_bytes (layout above).
 *   workspace:       device, cfg->workspace_bytes; receives every activation
 *                    the backward needs, and the status word (reset here).
 *   loss:            device fp32 scalar = mean per-position loss.
 *   token_loss:      device fp32 [batch*seq_len] or NULL.
 * Token/target ids outside [0, vocab) record GPT_EDATA (read it with
 * gpt_status); their rows are computed from id 0 and their loss is 0. */
int gpt_forward_loss(const gpt_config* cfg, const int32_t* tokens, const int32_t* targets,
                     const void* params, void* workspace, float* loss, float* token_loss,
                     void* stream);

/* Backward pass of the loss computed by the last gpt_forward_loss on the same
 * workspace and stream, with the same tokens/targets/params.
 *   grads:      device, same layout and dtype as params.
 *   accumulate: 0 = overwrite grads, 1 = grads += this step's gradient.
 * The gradient is that of the mean loss over all batch*seq_len positions. */
int gpt_backward(const gpt_config* cfg, const int32_t* tokens, const int32_t* targets,
                 const void* params, void* workspace, void* grads, int accumulate,
                 void* stream);

/* gpt_backward for data-parallel training ("ChatGPT'nizi 50 Dolara Nasil
 * Egitirsiniz?", section "Dagitilmis Egitim": the gradient exchange starts
 * while the backward still runs).
 *   grad_scale: every gradient is multiplied by it (> 0, finite).  With W
 *     replicas on equal batches, 1/W makes the sum of their gradients the
 *     gradient of the mean loss over all W*batch*seq_len positions.
 *   grad_ready_events: NULL, or n_events = n_layer + 2 CUDA events
 *     (cudaEvent_t, created by the caller on the current device), recorded on
 *     `stream` when a bucket of the gradient buffer is final: [0] lm_head,
 *     [1 + l] the four block matrices of layer l (recorded for l = n_layer-1
 *     down to 0, in that order), [n_layer + 1] wte.  A collective on another
 *     stream that waits for event i may then reduce that bucket while the
 *     backward goes on.
 * Everything else as gpt_backward (which is grad_scale 1, no events).
 * GPT_EINVAL for a bad scale, n_events != n_layer + 2 with events, or a NULL
 * event; GPT_ECUDA if an event record fails. */
int gpt_backward_ex(const gpt_config* cfg, const int32_t* tokens, const int32_t* targets,
                    const void* params, void* workspace, void* grads, int accumulate,
                    float grad_scale, void* const* grad_ready_events, int n_events, void* stream);

/* One whole training step from HOST token/target arrays (pinned memory gives
 * asynchronous copies): copies tokens/targets into the workspace's staging
 * area, runs gpt_forward_loss and gpt_backward, and copies the loss back to
 * *host_loss.  Returns after enqueueing; *host_loss is valid once `stream`
 * has been synchronised. */
int gpt_train_step_host(const gpt_config* cfg, const int32_t* host_tokens,
                        const int32_t* host_targets, const void* params, void* workspace,
                        void* grads, int accumulate, float* host_loss, void* stream);

/* Synchronise `stream`, then return the device status recorded in
 * `workspace` (GPT_OK or the first GPT_E* a kernel recorded), or GPT_ECUDA
 * if the synchronisation itself failed. */
int gpt_status(const void* workspace, void* stream);

/* Static string for a GPT_E* code. */
const char* gpt_strerror(int code);

/* Library version string. */
const char* gpt_version(void);

/* Embedding-gradient scatter-add without any device allocation.  No passage of
 * the pages corresponds to this call; it exists for callers that cannot
 * allocate device memory when they need the gradient (their device memory
 * all comes from a host framework's pool, or their memory budget is fixed up
 * front) and so cannot provide a gpt_config workspace either.
 *   tokens: device int32 [n_tokens];  dx0: device fp32 [n_tokens, d_model]
 *   (the gradient w.r.t. the gathered embeddings);  dwte: device [vocab,
 *   d_model], bf16 (dtype GPT_BF16) or fp32 (GPT_F32);  accumulate: 0 writes
 *   dwte (rows no token hits become 0), 1 adds to it.
 * Result: dwte[v] (+)= sum over positions n with tokens[n] == v of dx0[n],
 * summed in the same fixed order as the wte gradient of gpt_backward, so the
 * two agree bit for bit.  This call does not check the ids: the caller must
 * pass ids in [0, vocab) (gpt_forward_loss checks them, GPT_EDATA); an id
 * outside that range is summed into row 0 without any error.
 * Scratch: one 16 MiB array in device memory defined by the library, held by
 * every GPU that loads the library until the process exits.  The first call
 * in each CUDA context (keyed by the context's unique id) looks up that
 * array's device address (cudaGetSymbolAddress) with the context current;
 * make that first call before any stream capture.  All
 * calls share the array, so calls that may overlap on the same GPU (for
 * example on different streams) race: serialise them.  Sizes
 * whose scratch exceeds 16 MiB (about n_tokens * (8 + 8 d_model / 64) +
 * vocab * (4 n_tokens / 1024 + 28) bytes) return GPT_EUNSUPPORTED; NULL or
 * non-16-byte-aligned pointers GPT_EINVAL; enqueue failures GPT_ECUDA. */
int gpt_embedding_grad_noalloc(const int32_t* tokens, int64_t n_tokens, int32_t vocab,
                               int32_t d_model, int32_t dtype, const float* dx0, void* dwte,
                               int accumulate, void* stream);

/* Failure-path check (no counterpart on the pages): launches one kernel whose
 * single thread waits on a barrier that nothing arrives at, with the same
 * bounded wait (%globaltimer limit) that every pipeline kernel uses, here
 * limit_ns (1e3 .. 1e10) instead of 2 s.  When it expires the kernel records
 * GPT_ETIMEOUT in the workspace's status word (read with gpt_status) and
 * returns; nothing faults, traps or hangs, and the context stays usable.  The
 * next gpt_forward_loss clears the status word.  GPT_EINVAL for a NULL or
 * non-256-byte-aligned workspace or a limit out of range. */
int gpt_wait_expiry_check(void* workspace, int64_t limit_ns, void* stream);

/* ---- optimizer step ------------------------------------------------------------
 * "ChatGPT'nizi 50 Dolara Nasil Egitirsiniz?" (dev.to), section "2. Muon
 * Optimize Edici (nanochat/optim.py)": the embedding (wte) and lm_head are
 * updated with AdamW, every 2-D block matrix (Wqkv, Wo, Wup, Wdown) with Muon,
 * whose momentum is orthogonalised by the iteration
 *     A = X^T X,  B = b A + c A A,  X <- a X + X B
 * (the Gram matrix is taken over the smaller dimension: for a matrix with
 * fewer rows than columns, A = X X^T and X <- a X + B X).
 *
 * State (caller-owned, device, fp32, gpt_optim_state_bytes): three arrays of
 * the parameter buffer's element count, at the parameter buffer's element
 * offsets: the fp32 master weights, then m (AdamW first moment; Muon momentum),
 * then v (AdamW second moment; unused for Muon matrices).  The bf16 parameter
 * buffer is the master rounded to nearest even after every step: the pages'
 * layers cast a higher-precision weight to bf16 per call (section "3.
 * Hassasiyet Yonetimi").
 *
 * Per step, with t = step (1-based):
 *   AdamW:  m = b1 m + (1-b1) g;  v = b2 v + (1-b2) g^2;
 *           w = w (1 - lr wd) - lr (m / (1-b1^t)) / (sqrt(v / (1-b2^t)) + eps)
 *   Muon:   M = mu M + G;  U = G + mu M if nesterov else M;
 *           X = U / (||U||_F + 1e-7), then ns_steps iterations with
 *           (a, b, c) = ns_coeffs[i] in bf16 on the tensor cores;
 *           w = w - lr sqrt(max(1, rows/cols)) X.
 *   NorMuon (normuon = 1; the section's "NorMuon Varyans Azaltma" lines,
 *   whose undefined names are read after the published NorMuon method): per
 *   row r of X, v_mean = mean_c X^2; the row's state buf = beta2 buf +
 *   (1-beta2) v_mean (fp32, stored in the matrix's first `rows` v slots,
 *   zero after gpt_optim_init); step_r = 1/sqrt(max(buf, 1e-10)); X row r is
 *   scaled by step_r sqrt(sum v_mean) / max(sqrt(sum v_mean step^2), 1e-10)
 *   (the Frobenius norm of X is kept) before the update above.
 * bf16 configurations only (dtype GPT_F32 returns GPT_EUNSUPPORTED). */
typedef struct {
  float adam_lr, adam_beta1, adam_beta2, adam_eps, adam_weight_decay;
  float muon_lr, muon_momentum;
  int32_t muon_nesterov;   /* 1: orthogonalise G + mu M */
  int32_t ns_steps;        /* 0 .. 8 */
  float ns_coeffs[8][3];   /* (a, b, c) of iteration i */
  int64_t step;            /* AdamW step count t >= 1 */
  int32_t normuon;         /* 1: NorMuon row rescale of the orthogonalised update */
  float normuon_beta2;     /* its second-moment decay, in [0, 1) */
} gpt_optim;

/* Library defaults (the pages give no hyper-parameter values): AdamW lr 1e-3,
 * betas (0.9, 0.999), eps 1e-8 (Adam's published suggestions), no weight
 * decay; Muon lr 0.02, momentum 0.95, Nesterov; ns_steps 2 with the two
 * coefficient triples the page prints, (8.156, -22.483, 15.879) and
 * (4.043, -2.809, 0.5) (its list of five breaks off there: longer schedules
 * are the caller's); step 1; NorMuon off, its beta2 0.95 (the published
 * method's value).  Returns GPT_EINVAL for a NULL pointer. */
int gpt_optim_defaults(gpt_optim* opt);
/* Bytes of the optimizer state for an initialised config (3 fp32 copies of
 * the parameter buffer's elements). */
int gpt_optim_state_bytes(const gpt_config* cfg, size_t* bytes);
/* master = params (exact upcast), m = v = 0.  Async on `stream`. */
int gpt_optim_init(const gpt_config* cfg, const void* params, void* state, void* stream);
/* One optimizer step: updates state and params in place from grads (the
 * gradient buffer gpt_backward writes).  Its scratch (every layer's
 * Newton-Schulz iterates, stacked so that each product is one batched GEMM
 * over the layers) overwrites the layers' saved activations in the workspace:
 * a gpt_backward after it needs a new gpt_forward_loss first, as the new
 * parameters do anyway.  Async on `stream`, deterministic.  GPT_EINVAL for NULL or
 * misaligned pointers, ns_steps outside 0..8, step < 1, betas outside [0, 1)
 * (NorMuon's included, when on), normuon not 0 or 1, or non-finite
 * hyper-parameters. */
int gpt_optim_step(const gpt_config* cfg, const gpt_optim* opt, void* params, const void* grads,
                   void* state, void* workspace, void* stream);

/* ---- tracing (optional; per-launch CUDA events) ------------------------------
 * A trace records a CUDA event pair around every kernel launch that
 * gpt_forward_loss / gpt_backward / gpt_train_step_host make from the calling
 * host thread while the trace is attached, on the stream the kernels run on,
 * tagged with the kernel class below and the launch's algorithmic FLOPs and
 * HBM bytes (the minimum the operation must move).  The caller owns the trace;
 * recording stops silently once `capacity` launches are held (the count of
 * dropped launches is reported). */
#define GPT_K_GEMM 0      /* tensor-core (bf16) or SIMT (fp32) GEMM           */
#define GPT_K_ATTN_FWD 1  /* causal attention forward                         */
#define GPT_K_ATTN_BWD 2  /* causal attention backward (+QK-norm/RoPE bwd)    */
#define GPT_K_NORM 3      /* embedding gather + RMSNorm, RMSNorm fwd / bwd    */
#define GPT_K_QKV 4       /* RoPE + QK-norm + head-major scatter of q, k, v   */
#define GPT_K_LOSS 5      /* cross-entropy merge and loss mean                */
#define GPT_K_SORT 6      /* stable counting sort of positions by token id    */
#define GPT_K_SCATTER 7   /* embedding-gradient scatter-add                   */
#define GPT_K_OTHER 8     /* RoPE table, status reset                          */
#define GPT_K_QUANT 9     /* e4m3 quantization of projection operands (fp8)   */
#define GPT_K_COUNT 10

typedef struct gpt_trace gpt_trace;

typedef struct gpt_trace_stat {
  int32_t launches;  /* launcher calls recorded                               */
  int32_t kernels;   /* CUDA kernels (and memsets) those calls enqueued        */
  double ms;         /* summed event-pair durations                           */
  double flops;      /* summed algorithmic FLOPs                               */
  double bytes;      /* summed algorithmic HBM bytes                           */
} gpt_trace_stat;

/* Create a trace with room for `capacity` launches (creates 2*capacity CUDA
 * events on the current device). */
int gpt_trace_create(gpt_trace** trace, int capacity);
/* Attach `trace` to the calling host thread (NULL detaches). */
int gpt_trace_attach(gpt_trace* trace);
/* Forget every recorded launch (events are kept for reuse). */
int gpt_trace_reset(gpt_trace* trace);
/* Wait for the recorded events and fill stats[GPT_K_COUNT] (one per class);
 * *dropped receives the number of launches not recorded for lack of room. */
int gpt_trace_summary(gpt_trace* trace, gpt_trace_stat* stats, int32_t* dropped);

/* One recorded launch, in launch order. */
typedef struct gpt_trace_record {
  int32_t kind;      /* GPT_K_* */
  int32_t kernels;
  float ms;
  double flops;
  double bytes;
} gpt_trace_record;

/* Wait for the recorded events and copy up to `capacity` records, in launch
 * order, to `records`; *count receives the number copied. */
int gpt_trace_records(gpt_trace* trace, gpt_trace_record* records, int capacity, int32_t* count);
int gpt_trace_destroy(gpt_trace* trace);

#ifdef __cplusplus
}
#endif
#endif /* GPT_B200_H */
