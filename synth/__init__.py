"""Seeded synthetic workloads for the GPT training step.

This module is shared by the CPU oracle (``oracle/``), the tests and the
benchmark.  It holds the workload table (model shapes, batch shapes, seeds) and
the random generators for token streams and parameters, and nothing of the
model's arithmetic: no norm, no attention, no loss.  The training data the
pages train on (ClimbMix / FineWeb-EDU shards behind a 32,768-entry BPE
tokenizer, "ChatGPT'nizi 50 Dolara Nasil Egitirsiniz?", section "nanochat
Neleri Kapsar?"; TinyStories on the laptop page) is not available, so token ids
are drawn from a truncated Zipf law, which gives the embedding-gradient scatter
the heavy head (about 14 % of positions on id 0 at V=32768) that real BPE text
has.

Parameters follow the usual GPT initialisation: every matrix N(0, 0.02**2),
with the two residual-output projections (attention out-projection and MLP
down-projection) scaled by 1/sqrt(2*n_layer).  bf16 configurations round the
draws to bf16 (round to nearest even) once, here, so that every consumer sees
the same bytes.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Iterator, Tuple

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "workload",
    "param_shapes",
    "make_tokens",
    "make_params",
    "bf16_round",
    "bf16_bits_to_f64",
    "f64_to_bf16_bits",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One model + batch shape with the seeds that generate its inputs."""

    name: str
    n_layer: int
    d_model: int
    n_head: int
    head_dim: int
    d_ff: int
    vocab: int
    seq_len: int
    batch: int
    seed: int
    dtype: str  # "f32" or "bf16": storage type of parameters and activations
    tokens: str  # "uniform" (tokens and targets independent) or "zipf" (shifted stream)
    zipf_s: float = 1.1
    rope_base: float = 10000.0
    norm_eps: float = 1e-6
    qk_norm: bool = True
    n_kv_head: int = 0  # key/value heads (GQA); 0 = n_head
    window: int = 0     # sliding attention window in positions; 0 = full causal
    fp8: bool = False   # e4m3 operands in the forward block projections
    ve_every: int = 0   # value embeddings on layers l % ve_every == ve_every - 1; 0 = none
    ve_gate_channels: int = 32
    resid_lambdas: bool = False  # per-layer residual scaling x = a x + b x0
    smear: bool = False          # previous-token embedding mixing after the gather
    backout: bool = False        # subtract the middle layer's residual before the final norm

    @property
    def n_tokens(self) -> int:
        return self.batch * self.seq_len

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny fp32 decoder, the laptop story-model shape, and
# the depth dial at 4, 12 and 24 (d_model = 64*depth, head_dim = 128, d_ff = 4*d).
WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny", 2, 64, 4, 16, 256, 256, 64, 4, 0, "f32", "uniform"),
        Workload("story", 3, 256, 4, 64, 1024, 4096, 256, 32, 1, "bf16", "zipf"),
        Workload("d4", 4, 256, 2, 128, 1024, 32768, 512, 8, 2, "bf16", "zipf"),
        Workload("d12", 12, 768, 6, 128, 3072, 32768, 2048, 16, 3, "bf16", "zipf"),
        Workload("d24", 24, 1536, 12, 128, 6144, 32768, 2048, 16, 4, "bf16", "zipf"),
    ]
}


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.replace(**overrides) if overrides else w


def param_shapes(w: Workload) -> Iterator[Tuple[str, Tuple[int, int]]]:
    """Parameter names and [out, in] shapes, in generation order."""
    d, f, v = w.d_model, w.d_ff, w.vocab
    qkv = d + 2 * (w.n_kv_head or w.n_head) * w.head_dim
    yield "wte", (v, d)
    for l in range(w.n_layer):
        yield f"layers.{l}.wqkv", (qkv, d)
        yield f"layers.{l}.wo", (d, d)
        yield f"layers.{l}.wup", (f, d)
        yield f"layers.{l}.wdown", (d, f)
    yield "lm_head", (v, d)
    # block-variant parameters, after the base model's (their draws come last)
    kv = (w.n_kv_head or w.n_head) * w.head_dim
    if w.ve_every:
        for l in range(w.n_layer):
            if l % w.ve_every == w.ve_every - 1:
                yield f"ve.{l}", (v, kv)
                yield f"ve_gate.{l}", (w.n_kv_head or w.n_head, w.ve_gate_channels)
    if w.resid_lambdas:
        yield "lambdas", (w.n_layer, 2)          # [resid, x0] per layer
    if w.smear:
        yield "smear_gate", (1, 24)
    if w.smear or w.backout:
        yield "scalars", (1, 2)                  # [smear lambda, backout lambda]


# Draws of the block-variant parameters: (mean, scale) of a normal law per
# kind; their initial values are the caller's, these only make every term of
# the variants visible in the tests' gradients.
_VARIANT_DRAWS = {"ve": (0.0, 0.3), "ve_gate": (0.0, 0.5), "smear_gate": (0.0, 10.0)}


# ---------------------------------------------------------------------------
# bf16 helpers (storage format only)
# ---------------------------------------------------------------------------

def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round to bf16 (nearest, ties to even) via fp32; returns uint16 bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = (u + 0x7FFF + lsb) >> 16
    # NaN stays NaN (none are generated here, kept for completeness)
    nan = np.isnan(f)
    out = rounded.astype(np.uint16)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def bf16_round(x: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f64(f64_to_bf16_bits(x))


# ---------------------------------------------------------------------------
# token streams
# ---------------------------------------------------------------------------

def _zipf_ids(rng: np.random.Generator, vocab: int, s: float, size) -> np.ndarray:
    """P(id = k-1) proportional to k**-s for k = 1..vocab, by inverse CDF."""
    k = np.arange(1, vocab + 1, dtype=np.float64)
    cdf = np.cumsum(k ** (-s))
    cdf /= cdf[-1]
    u = rng.random(size)
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, vocab - 1).astype(np.int32)


def make_tokens(w: Workload) -> Tuple[np.ndarray, np.ndarray]:
    """int32 tokens and targets, both [batch, seq_len]."""
    rng = np.random.Generator(np.random.PCG64(w.seed))
    if w.tokens == "uniform":
        tok = rng.integers(0, w.vocab, size=(w.batch, w.seq_len), dtype=np.int64)
        tgt = rng.integers(0, w.vocab, size=(w.batch, w.seq_len), dtype=np.int64)
        return tok.astype(np.int32), tgt.astype(np.int32)
    if w.tokens == "zipf":
        stream = _zipf_ids(rng, w.vocab, w.zipf_s, (w.batch, w.seq_len + 1))
        return (np.ascontiguousarray(stream[:, :-1]), np.ascontiguousarray(stream[:, 1:]))
    raise ValueError(f"unknown token law {w.tokens!r}")


# ---------------------------------------------------------------------------
# parameters
# ---------------------------------------------------------------------------

def make_params(w: Workload, as_bits: bool = False) -> Dict[str, np.ndarray]:
    """Seeded parameters.

    Returns float64 arrays holding exactly the stored values (bf16-rounded for
    bf16 workloads, fp32-rounded for f32 ones).  With ``as_bits`` and a bf16
    workload, returns the uint16 bit patterns instead (what a device buffer
    holds); with ``as_bits`` and an f32 workload, float32 arrays.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed + 1000))
    out_scale = 1.0 / math.sqrt(2.0 * w.n_layer) if w.n_layer > 0 else 1.0
    params: Dict[str, np.ndarray] = {}
    for name, shape in param_shapes(w):
        x = rng.standard_normal(shape, dtype=np.float32) * np.float32(0.02)
        if name.endswith(".wo") or name.endswith(".wdown"):
            x = x * np.float32(out_scale)
        kind = name.split(".")[0]
        if kind in _VARIANT_DRAWS:
            mean, scale = _VARIANT_DRAWS[kind]
            x = x * np.float32(scale / 0.02) + np.float32(mean)
        elif name == "lambdas":   # resid near 1, x0 near 0
            x = x * np.float32(5.0) + np.array([1.0, 0.0], dtype=np.float32)
        elif name == "scalars":   # smear and backout lambdas near 0.5 and 0.3
            x = x * np.float32(5.0) + np.array([0.5, 0.3], dtype=np.float32)
        if w.dtype == "bf16":
            bits = f64_to_bf16_bits(x)
            params[name] = bits if as_bits else bf16_bits_to_f64(bits)
        elif w.dtype == "f32":
            params[name] = x.astype(np.float32) if as_bits else x.astype(np.float64)
        else:
            raise ValueError(w.dtype)
    return params

def random_bf16_bits(shape, seed: int, scale: float) -> np.ndarray:
    """Seeded N(0, scale^2) values rounded to bf16 (uint16 bit patterns): the
    synthetic gradients fed to the optimizer step."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal(shape, dtype=np.float32) * np.float32(scale)
    return f64_to_bf16_bits(x)
