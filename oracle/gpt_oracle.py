"""fp64 CPU oracle for one forward + backward training step of the GPT.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check in
``__graft_entry__`` and the ``cpu_baseline`` / reference arm of ``bench.py``
may import this module.  The CUDA library never calls it, and it never calls
the CUDA library: the two share no code.  Inputs come from ``synth`` (seeded
generators, no model arithmetic).

What is computed, and where it comes from
-----------------------------------------
"ChatGPT'nizi 50 Dolara Nasil Egitirsiniz?" (dev.to), section "1. GPT Modeli
(nanochat/gpt.py)", lists the model's ingredients: rotary embeddings, QK
normalisation, untied embedding and output weights, the ReLU^2 activation,
grouped-query attention (GQA) and sliding-window attention (Flash Attention 3
is how the page runs the attention, which changes nothing in exact
arithmetic).
Section "3. Hassasiyet Yonetimi (nanochat/common.py)" shows every linear layer
as ``F.linear(x, W)`` with W stored [out, in] and no bias.  Section "5. Flash
Dikkat Mekanizmasi Birlesimi" calls the attention with ``causal=True``.  The
norm is parameter-free RMSNorm and the loss is the mean next-token
cross-entropy in fp32 or better.

Where the pages are silent the plainest reading is taken:

* pre-norm blocks (norm before attention and before the MLP), one final norm
  before lm_head, no norm directly after the embedding;
* RMSNorm y = x / sqrt(mean(x^2) + eps), eps = 1e-6, no weight;
* RoPE on q and k with half-split pairs (i, i + hd/2), angle t * base^(-2i/hd),
  (a, b) -> (a cos - b sin, a sin + b cos), positions 0..T-1 per sequence;
* QK norm = the same parameter-free RMSNorm over each head's hd entries,
  applied after RoPE (a rotation keeps the norm, so the order does not change
  the result in exact arithmetic);
* attention scale 1/sqrt(hd), no dropout, no soft-capping;
* GQA: ``n_kv_head`` key/value heads shared by ``n_head / n_kv_head``
  consecutive query heads (query head h reads key/value head
  h // (n_head / n_kv_head)); 0 or n_head is ordinary multi-head attention;
* sliding window: section "5. Flash Dikkat Mekanizmasi Birlesimi" passes a
  ``window_size`` to the causal attention call; with ``window`` = W >= 1 query
  i sees keys j with i - W < j <= i (its W most recent positions, itself
  included), in every layer; 0 is the full causal window;
* MLP u = h W_up^T, a = max(u, 0)^2, y = a W_down^T (not gated);
* loss = mean over all B*T positions of logsumexp(z) - z[target].

FP8 (``fp8``; the page's training command line has an ``--fp8`` flag and
names no scaling recipe).  Reading taken: the four block projections (W_qkv,
W_o, W_up, W_down) multiply e4m3 operands in the forward and in their data
gradients dX = dY W; the embedding, lm_head and every weight gradient stay as
above.

* quantizer input: the operand as the bf16 value the GPU stores (activations
  rounded to bf16 here, weights are bf16 already) -- the same precision in
  which the kernel takes its rounding decision;
* scales: one per activation row (token), one per weight tensor, each the
  largest power of two 2^k with amax * 2^k <= 448 (e4m3's largest finite
  value; k = 0 for an all-zero row), so scaling and unscaling are exact;
* code: round to the nearest e4m3 value (OCP E4M3: 4 exponent bits, bias 7,
  3 mantissa bits, subnormals, no infinities), ties to the even code;
* product: the dequantized operands multiplied exactly (fp64 here);
* data gradient: dX = dY W with dY through e4m3 exactly as an activation
  (rounded to bf16, one power-of-two scale per row, i.e. per token) and W
  through the forward's per-tensor codes;
* weight gradient: dW = dY^T X with the unquantized dY and X (the bf16
  model's, at the FP8 forward's activations), i.e. the quantizer taken as the
  identity there (straight-through).

Block variants (section "1. GPT Modeli": the "Deger Gommeleri (ResFormer)"
and "Verimlilik Puf Noktalari" listings).  The page prints each as a line or
two; the widths, the layers they act on and the initial values are not
printed.  Readings taken (every scale and gate is a parameter, so its initial
value is the caller's):

* value embeddings (``ve_every`` = k >= 1): layers l with l % k == k - 1 own a
  table VE_l [vocab, n_kv_head*hd]; with h the block's normalised input (the
  attention's input), gate = 3 sigmoid(h[:, :C] W_g^T), W_g [n_kv_head, C],
  C = ``ve_gate_channels``, and v <- v + gate (per key/value head) * VE_l[tok];
* per-layer residual scaling (``resid_lambdas``): on entering layer l,
  x <- lam[l, 0] x + lam[l, 1] x0, with x0 the stream entering layer 0;
* smear (``smear``), once, right after the embedding gather e = wte[tok]:
  g_t = smear_lambda sigmoid(e_t[:24] . w_smear), x_t = e_t + g_t e_{t-1}
  (e_{-1} = 0: the first position of a sequence mixes nothing);
* backout (``backout``): x_b is the stream entering layer n_layer // 2 (after
  its residual scaling); after the last layer x <- x - backout_lambda x_b,
  then the final norm.

Layout conventions shared with the library's documented ABI (not its code):
W_qkv is [(n_head + 2 n_kv_head) hd, d] with the q rows first, then k, then v
([3d, d] without GQA); inside each block head h owns rows [h*hd, (h+1)*hd).

The backward pass is derived by hand from the forward above; each step names
the forward step it inverts.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Sequence

import numpy as np

__all__ = [
    "OracleConfig",
    "from_workload",
    "rms_norm",
    "rms_norm_backward",
    "rope_tables",
    "rope",
    "rope_backward",
    "attention_mask",
    "causal_attention",
    "causal_attention_backward",
    "cross_entropy",
    "e4m3_round",
    "pow2_exponent",
    "fp8_rows",
    "fp8_tensor",
    "fp8_linear",
    "fp8_weights",
    "sequence_forward",
    "sequence_backward",
    "step",
    "StepResult",
]


@dataclasses.dataclass(frozen=True)
class OracleConfig:
    n_layer: int
    d_model: int
    n_head: int
    head_dim: int
    d_ff: int
    vocab: int
    seq_len: int
    batch: int
    norm_eps: float = 1e-6
    rope_base: float = 10000.0
    qk_norm: bool = True
    n_kv_head: int = 0   # 0: n_head (multi-head attention)
    window: int = 0      # 0: full causal window
    fp8: bool = False    # e4m3 operands in the block projections' forward
    ve_every: int = 0    # value embeddings on layers l % ve_every == ve_every - 1; 0: none
    ve_gate_channels: int = 32
    resid_lambdas: bool = False
    smear: bool = False
    backout: bool = False

    @property
    def kv_heads(self) -> int:
        return self.n_kv_head or self.n_head

    def has_ve(self, l: int) -> bool:
        return self.ve_every > 0 and l % self.ve_every == self.ve_every - 1

    @property
    def backout_layer(self) -> int:
        return self.n_layer // 2


def from_workload(w) -> OracleConfig:
    return OracleConfig(
        n_layer=w.n_layer, d_model=w.d_model, n_head=w.n_head, head_dim=w.head_dim,
        d_ff=w.d_ff, vocab=w.vocab, seq_len=w.seq_len, batch=w.batch,
        norm_eps=w.norm_eps, rope_base=w.rope_base, qk_norm=w.qk_norm,
        n_kv_head=getattr(w, "n_kv_head", 0), window=getattr(w, "window", 0),
        fp8=bool(getattr(w, "fp8", False)), ve_every=getattr(w, "ve_every", 0),
        ve_gate_channels=getattr(w, "ve_gate_channels", 32),
        resid_lambdas=bool(getattr(w, "resid_lambdas", False)),
        smear=bool(getattr(w, "smear", False)), backout=bool(getattr(w, "backout", False)))


def _sigmoid(z: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-z))


SMEAR_CHANNELS = 24  # the smear gate reads x[:, :, :24] ("Verimlilik Puf Noktalari")


# ---------------------------------------------------------------------------
# building blocks
# ---------------------------------------------------------------------------

def rms_norm(x: np.ndarray, eps: float):
    """Parameter-free RMSNorm over the last axis.

    Returns (y, r) with r = 1/sqrt(mean(x^2) + eps) (one per row) and y = x*r.
    """
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r, r


def rms_norm_backward(dy: np.ndarray, y: np.ndarray, r: np.ndarray) -> np.ndarray:
    """Inverse of ``rms_norm``: dx = r * (dy - y * mean(dy * y)).

    From y_i = x_i r with dr/dx_j = -r^3 x_j / n.
    """
    return r * (dy - y * np.mean(dy * y, axis=-1, keepdims=True))


def rope_tables(seq_len: int, head_dim: int, base: float):
    """cos/sin of t * base^(-2i/hd) for t < seq_len, i < hd/2, shape [T, hd/2]."""
    half = head_dim // 2
    i = np.arange(half, dtype=np.float64)
    theta = base ** (-2.0 * i / head_dim)
    ang = np.arange(seq_len, dtype=np.float64)[:, None] * theta[None, :]
    return np.cos(ang), np.sin(ang)


def rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate each (x[i], x[i+hd/2]) pair of x [T, H, hd] by the position's angle."""
    half = x.shape[-1] // 2
    a, b = x[..., :half], x[..., half:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def rope_backward(dy: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Transpose of the rotation in ``rope`` (rotation by the negative angle)."""
    half = dy.shape[-1] // 2
    da, db = dy[..., :half], dy[..., half:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([da * c + db * s, -da * s + db * c], axis=-1)


def _heads_first(x: np.ndarray) -> np.ndarray:
    """[T, H, hd] -> [H, T, hd]"""
    return np.ascontiguousarray(x.transpose(1, 0, 2))


def attention_mask(T: int, window: int = 0) -> np.ndarray:
    """[T, T] bool, True where query i may attend to key j: j <= i, and
    i - j < window when a window is set (window >= 1)."""
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    visible = j <= i
    if window > 0:
        visible &= (i - j) < window
    return visible


def _per_query_head(x: np.ndarray, n_head: int) -> np.ndarray:
    """[T, Hkv, hd] key/value heads -> [T, n_head, hd]: query head h uses
    key/value head h // (n_head / Hkv)."""
    return np.repeat(x, n_head // x.shape[1], axis=1)


def _causal_probs(q: np.ndarray, k: np.ndarray, window: int):
    """Scores and probabilities for q, k [T, H, hd]; returns P [H, T, T] and lse [H, T]."""
    T, H, hd = q.shape
    s = (_heads_first(q) @ _heads_first(k).transpose(0, 2, 1)) / math.sqrt(hd)
    s = np.where(attention_mask(T, window)[None, :, :], s, -np.inf)
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    tot = np.sum(e, axis=-1, keepdims=True)
    return e / tot, (m + np.log(tot))[..., 0]


def causal_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, window: int = 0):
    """softmax(q k^T / sqrt(hd), masked by ``attention_mask``) v, per query head.

    q: [T, H, hd]; k, v: [T, Hkv, hd] with Hkv dividing H (GQA).  Returns
    o [T, H, hd], the probabilities P [H, T, T] and the row log-sum-exp [H, T]
    of the scaled, masked scores.
    """
    H = q.shape[1]
    p, lse = _causal_probs(q, _per_query_head(k, H), window)
    o = (p @ _heads_first(_per_query_head(v, H))).transpose(1, 0, 2)
    return o, p, lse


def causal_attention_backward(do, q, k, v, p):
    """Gradients of ``causal_attention`` w.r.t. q, k, v given dO and P.

    dV = P^T dO;  dP = dO V^T;  dS = P * (dP - rowsum(dP * P));
    dQ = dS K / sqrt(hd);  dK = dS^T Q / sqrt(hd), per query head; a shared
    key/value head (GQA) receives the sum over the query heads that read it.
    The mask is already in P (masked entries are exactly 0).
    """
    T, H, hd = q.shape
    Hkv = k.shape[1]
    do_h, q_h = _heads_first(do), _heads_first(q)
    k_h, v_h = _heads_first(_per_query_head(k, H)), _heads_first(_per_query_head(v, H))
    dv = p.transpose(0, 2, 1) @ do_h
    dp = do_h @ v_h.transpose(0, 2, 1)
    ds = p * (dp - np.sum(dp * p, axis=-1, keepdims=True))
    dq = (ds @ k_h) / math.sqrt(hd)
    dk = (ds.transpose(0, 2, 1) @ q_h) / math.sqrt(hd)
    back = lambda t: t.transpose(1, 0, 2)
    group = lambda t: back(t).reshape(T, Hkv, H // Hkv, hd).sum(axis=2)
    return back(dq), group(dk), group(dv)


# ---------------------------------------------------------------------------
# FP8 (e4m3) forward projections
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def _e4m3_table():
    """Every finite non-negative e4m3 value (codes 0x00..0x7E) in increasing
    order: exponent field e, mantissa m -> (m/8) 2^-6 if e == 0, else
    (1 + m/8) 2^(e-7).  Code 0x7F is NaN."""
    codes = np.arange(0x7F)
    e, m = codes >> 3, codes & 7
    vals = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    return vals, codes


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """x rounded to the nearest e4m3 value, ties to the even code (|x| <= 448)."""
    vals, codes = _e4m3_table()
    a = np.abs(x)
    hi_i = np.clip(np.searchsorted(vals, a), 1, len(vals) - 1)
    lo, hi = vals[hi_i - 1], vals[hi_i]
    up = (hi - a < a - lo) | ((hi - a == a - lo) & (codes[hi_i] % 2 == 0))
    return np.sign(x) * np.where(up, hi, lo)


def pow2_exponent(amax: np.ndarray) -> np.ndarray:
    """The largest k with amax * 2^k <= 448 (0 where amax == 0), elementwise."""
    amax = np.asarray(amax, dtype=np.float64)
    safe = np.where(amax > 0, amax, 1.0)
    _, e = np.frexp(E4M3_MAX / safe)       # 448/amax = f 2^e, f in [0.5, 1)
    k = e.astype(np.int64) - 1
    k = np.where(np.ldexp(safe, k) > E4M3_MAX, k - 1, k)     # exact fix-ups
    k = np.where(np.ldexp(safe, k + 1) <= E4M3_MAX, k + 1, k)
    return np.where(amax > 0, k, 0)


def _round_bf16(x: np.ndarray) -> np.ndarray:
    """Nearest bf16 value (ties to even), through the fp32 bit pattern."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def fp8_rows(x: np.ndarray) -> np.ndarray:
    """The value an activation x [R, K] takes through e4m3: rounded to bf16,
    scaled per row by a power of two, coded, unscaled."""
    xb = _round_bf16(x)
    kx = pow2_exponent(np.max(np.abs(xb), axis=1))
    return np.ldexp(e4m3_round(np.ldexp(xb, kx[:, None])), -kx[:, None])


def fp8_tensor(w: np.ndarray) -> np.ndarray:
    """The value a weight W (bf16 values) takes through e4m3 with one
    power-of-two scale for the whole tensor."""
    kw = pow2_exponent(np.max(np.abs(w)))
    return np.ldexp(e4m3_round(np.ldexp(w, kw)), -kw)


def fp8_linear(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """x W^T with both operands in e4m3: x [R, K] scaled per row, W [N, K]
    (bf16 values) per tensor, by powers of two; the product is exact in fp64."""
    return fp8_rows(x) @ fp8_tensor(w).T


def _linear(cfg: "OracleConfig", x: np.ndarray, w: np.ndarray,
            w_fp8: Optional[np.ndarray] = None) -> np.ndarray:
    """One block projection, x W^T (F.linear without bias); with fp8, the
    e4m3 operands (w_fp8: W through e4m3, when already computed)."""
    if not cfg.fp8:
        return x @ w.T
    return fp8_rows(x) @ (fp8_tensor(w) if w_fp8 is None else w_fp8).T


def _dgrad(dy: np.ndarray, w: np.ndarray, w_fp8: Optional[np.ndarray]) -> np.ndarray:
    """The data gradient of one block projection y = x W^T: dy W, or with
    fp8 (w_fp8: W through e4m3) dy through e4m3 per row times w_fp8."""
    if w_fp8 is None:
        return dy @ w
    return fp8_rows(dy) @ w_fp8


def fp8_weights(cfg: "OracleConfig", params: Dict[str, np.ndarray]) -> Optional[Dict[str, np.ndarray]]:
    """Every block matrix through e4m3 (fp8 configs; None otherwise): the
    same for every sequence of a step, so computed once per step."""
    if not cfg.fp8:
        return None
    names = [f"layers.{l}.{m}" for l in range(cfg.n_layer) for m in ("wqkv", "wo", "wup", "wdown")]
    return {n: fp8_tensor(params[n]) for n in names}


def cross_entropy(z: np.ndarray, y: np.ndarray):
    """Per-position loss logsumexp(z) - z[y] (max-shifted), plus lse and softmax."""
    m = np.max(z, axis=-1, keepdims=True)
    e = np.exp(z - m)
    tot = np.sum(e, axis=-1, keepdims=True)
    lse = (m + np.log(tot))[:, 0]
    loss = lse - z[np.arange(z.shape[0]), y]
    return loss, lse, e / tot


# ---------------------------------------------------------------------------
# one sequence
# ---------------------------------------------------------------------------

def _layer_params(params, l):
    return (params[f"layers.{l}.wqkv"], params[f"layers.{l}.wo"],
            params[f"layers.{l}.wup"], params[f"layers.{l}.wdown"])


def sequence_forward(cfg: OracleConfig, params: Dict[str, np.ndarray],
                     tok: np.ndarray, tgt: np.ndarray,
                     w_fp8: Optional[Dict[str, np.ndarray]] = None) -> dict:
    """Forward pass of one sequence (tok, tgt: int [T]); returns a cache dict.

    The cache holds what the backward needs plus the per-position loss
    (``token_loss``), the final logits' lse, and per-layer intermediates.
    """
    T = tok.shape[0]
    d, H, hd, Hkv = cfg.d_model, cfg.n_head, cfg.head_dim, cfg.kv_heads
    dkv = Hkv * hd
    eps = cfg.norm_eps
    if w_fp8 is None:
        w_fp8 = fp8_weights(cfg, params)
    wq = (lambda name: w_fp8[name]) if w_fp8 is not None else (lambda name: None)
    cos, sin = rope_tables(T, hd, cfg.rope_base)

    x = params["wte"][tok].astype(np.float64)           # token embedding gather
    smear = None
    if cfg.smear:                                        # mix in the previous token's embedding
        e = x
        u = e[:, :SMEAR_CHANNELS] @ params["smear_gate"][0]
        sg = _sigmoid(u)
        prev = np.zeros_like(e)
        prev[1:] = e[:-1]
        x = e + (params["scalars"][0, 0] * sg)[:, None] * prev
        smear = dict(e=e, sg=sg, prev=prev)
    x0 = x
    x_b = None
    layers = []
    for l in range(cfg.n_layer):
        wqkv, wo, wup, wdown = _layer_params(params, l)
        c = {}
        if cfg.resid_lambdas:                            # per-layer residual scaling
            c["x_prev"] = x
            x = params["lambdas"][l, 0] * x + params["lambdas"][l, 1] * x0
        if cfg.backout and l == cfg.backout_layer:
            x_b = x
        c["x_in"] = x
        h, r1 = rms_norm(x, eps)                         # pre-attention norm
        qkv = _linear(cfg, h, wqkv, wq(f"layers.{l}.wqkv"))  # F.linear, no bias
        q = qkv[:, :d].reshape(T, H, hd)
        k = qkv[:, d:d + dkv].reshape(T, Hkv, hd)
        v = qkv[:, d + dkv:].reshape(T, Hkv, hd)
        if cfg.has_ve(l):                                # value embedding, gated per kv head
            C = cfg.ve_gate_channels
            gz = h[:, :C] @ params[f"ve_gate.{l}"].T     # [T, Hkv]
            gate = 3.0 * _sigmoid(gz)
            ve = params[f"ve.{l}"][tok].reshape(T, Hkv, hd)
            v = v + gate[:, :, None] * ve
            c.update(ve_gz=gz, ve_rows=ve)
        q = rope(q, cos, sin)
        k = rope(k, cos, sin)
        if cfg.qk_norm:
            qn, rq = rms_norm(q, eps)
            kn, rk = rms_norm(k, eps)
        else:
            qn, rq, kn, rk = q, None, k, None
        o, p, lse = causal_attention(qn, kn, v, cfg.window)
        o2 = o.reshape(T, d)
        x = x + _linear(cfg, o2, wo, wq(f"layers.{l}.wo"))  # attention residual
        x_mid = x
        h2, r2 = rms_norm(x, eps)                        # pre-MLP norm
        u = _linear(cfg, h2, wup, wq(f"layers.{l}.wup"))
        a = np.maximum(u, 0.0) ** 2                      # ReLU^2
        x = x + _linear(cfg, a, wdown, wq(f"layers.{l}.wdown"))  # MLP residual
        c.update(h=h, r1=r1, q=q, k=k, qn=qn, kn=kn, rq=rq, rk=rk, v=v, o=o2,
                 lse=lse, x_mid=x_mid, h2=h2, r2=r2, u=u, a=a)
        layers.append(c)

    if cfg.backout:                                      # take out the middle layers' residual
        x = x - params["scalars"][0, 1] * x_b
    hf, rf = rms_norm(x, eps)                            # final norm
    z = hf @ params["lm_head"].T                         # untied lm_head
    loss_t, lse_z, probs = cross_entropy(z, tgt)
    return {"tok": tok, "tgt": tgt, "layers": layers, "x_out": x, "hf": hf,
            "rf": rf, "z": z, "probs": probs, "lse_z": lse_z, "token_loss": loss_t,
            "cos": cos, "sin": sin, "x0": x0, "x_b": x_b, "smear": smear}


def sequence_backward(cfg: OracleConfig, params: Dict[str, np.ndarray], cache: dict,
                      scale: float, grads: Dict[str, np.ndarray],
                      w_fp8: Optional[Dict[str, np.ndarray]] = None) -> None:
    """Accumulate d(scale * sum_t loss_t)/d(params) into ``grads``; with fp8,
    ``w_fp8`` holds the block matrices through e4m3 (``fp8_weights``)."""
    tok, tgt = cache["tok"], cache["tgt"]
    T = tok.shape[0]
    d, H, hd, Hkv = cfg.d_model, cfg.n_head, cfg.head_dim, cfg.kv_heads
    cos, sin = cache["cos"], cache["sin"]

    g = cache["probs"].copy()                            # d loss / d z
    g[np.arange(T), tgt] -= 1.0
    g *= scale
    grads["lm_head"] += g.T @ cache["hf"]
    dhf = g @ params["lm_head"]
    dx = rms_norm_backward(dhf, cache["hf"], cache["rf"])
    dx_final = dx                                        # backout: x_out = x_L - beta x_b
    if cfg.backout:
        grads["scalars"][0, 1] -= np.sum(dx_final * cache["x_b"])
    dx0 = np.zeros_like(dx)                              # residual scaling's x0 term

    if cfg.fp8 and w_fp8 is None:
        w_fp8 = fp8_weights(cfg, params)
    wq = (lambda name: w_fp8[name]) if cfg.fp8 else (lambda name: None)
    for l in reversed(range(cfg.n_layer)):
        wqkv, wo, wup, wdown = _layer_params(params, l)
        c = cache["layers"][l]
        # x_out = x_mid + a W_down^T
        grads[f"layers.{l}.wdown"] += dx.T @ c["a"]
        da = _dgrad(dx, wdown, wq(f"layers.{l}.wdown"))
        du = da * 2.0 * np.maximum(c["u"], 0.0)
        grads[f"layers.{l}.wup"] += du.T @ c["h2"]
        dh2 = _dgrad(du, wup, wq(f"layers.{l}.wup"))
        dx = dx + rms_norm_backward(dh2, c["h2"], c["r2"])
        # x_mid = x_in + o W_o^T
        grads[f"layers.{l}.wo"] += dx.T @ c["o"]
        do = _dgrad(dx, wo, wq(f"layers.{l}.wo")).reshape(T, H, hd)
        _, p, _ = causal_attention(c["qn"], c["kn"], c["v"], cfg.window)
        dqn, dkn, dv = causal_attention_backward(do, c["qn"], c["kn"], c["v"], p)
        dh_ve = None
        if cfg.has_ve(l):                                # v = v_proj + gate * VE[tok]
            C = cfg.ve_gate_channels
            sg = _sigmoid(c["ve_gz"])
            gate = 3.0 * sg
            np.add.at(grads[f"ve.{l}"], tok, (gate[:, :, None] * dv).reshape(T, Hkv * hd))
            dgz = np.sum(dv * c["ve_rows"], axis=2) * 3.0 * sg * (1.0 - sg)   # [T, Hkv]
            grads[f"ve_gate.{l}"] += dgz.T @ c["h"][:, :C]
            dh_ve = np.zeros((T, d))
            dh_ve[:, :C] = dgz @ params[f"ve_gate.{l}"]
        if cfg.qk_norm:
            dq = rms_norm_backward(dqn, c["qn"], c["rq"])
            dk = rms_norm_backward(dkn, c["kn"], c["rk"])
        else:
            dq, dk = dqn, dkn
        dq = rope_backward(dq, cos, sin)
        dk = rope_backward(dk, cos, sin)
        dqkv = np.concatenate([dq.reshape(T, d), dk.reshape(T, Hkv * hd), dv.reshape(T, Hkv * hd)],
                              axis=1)
        grads[f"layers.{l}.wqkv"] += dqkv.T @ c["h"]
        dh = _dgrad(dqkv, wqkv, wq(f"layers.{l}.wqkv"))
        if dh_ve is not None:
            dh = dh + dh_ve
        dx = dx + rms_norm_backward(dh, c["h"], c["r1"])
        if cfg.backout and l == cfg.backout_layer:       # x_b is this layer's input
            dx = dx - params["scalars"][0, 1] * dx_final
        if cfg.resid_lambdas:                            # x_in = a x_prev + b x0
            a, b = params["lambdas"][l, 0], params["lambdas"][l, 1]
            grads["lambdas"][l, 0] += np.sum(dx * c["x_prev"])
            grads["lambdas"][l, 1] += np.sum(dx * cache["x0"])
            dx0 = dx0 + b * dx
            dx = a * dx

    dx = dx + dx0                                        # x0 is the stream entering layer 0
    if cfg.smear:                                        # x = e + g * prev(e), g = beta sigmoid(u)
        sm = cache["smear"]
        lam = params["scalars"][0, 0]
        dg = np.sum(dx * sm["prev"], axis=1)             # [T]
        grads["scalars"][0, 0] += np.sum(dg * sm["sg"])
        du = dg * lam * sm["sg"] * (1.0 - sm["sg"])
        grads["smear_gate"][0] += du @ sm["e"][:, :SMEAR_CHANNELS]
        de = dx.copy()
        de[:-1] += (lam * sm["sg"][1:])[:, None] * dx[1:]   # e_t feeds x_{t+1} through prev
        de[:, :SMEAR_CHANNELS] += du[:, None] * params["smear_gate"][0][None, :]
        dx = de

    np.add.at(grads["wte"], tok, dx)                     # embedding scatter-add


# ---------------------------------------------------------------------------
# the whole step
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class StepResult:
    loss: float
    token_loss: np.ndarray                 # [B, T] (only the rows that were run)
    grads: Optional[Dict[str, np.ndarray]]
    caches: Optional[list] = None


def step(cfg: OracleConfig, params: Dict[str, np.ndarray], tokens: np.ndarray,
         targets: np.ndarray, *, backward: bool = True, keep_caches: bool = False,
         rows: Optional[Sequence[int]] = None, loss_denominator: Optional[int] = None
         ) -> StepResult:
    """Loss = mean over all B*T positions; gradients of that loss.

    Sequences are independent, so they are run one at a time and their
    gradient contributions summed.  ``rows`` restricts the run to some
    sequences (their token losses, and their share of the gradient with the
    full batch's 1/(B*T) factor); ``loss_denominator`` overrides B*T.
    """
    B, T = tokens.shape
    denom = loss_denominator if loss_denominator is not None else B * T
    rows = list(range(B)) if rows is None else list(rows)
    w_fp8 = fp8_weights(cfg, params)
    grads = None
    if backward:
        grads = {name: np.zeros_like(p, dtype=np.float64) for name, p in params.items()}
    token_loss = np.zeros((len(rows), T))
    caches = [] if keep_caches else None
    for i, b in enumerate(rows):
        cache = sequence_forward(cfg, params, tokens[b], targets[b], w_fp8)
        token_loss[i] = cache["token_loss"]
        if backward:
            sequence_backward(cfg, params, cache, 1.0 / denom, grads, w_fp8)
        if keep_caches:
            caches.append(cache)
    loss = float(np.sum(token_loss) / denom)
    return StepResult(loss=loss, token_loss=token_loss, grads=grads, caches=caches)
