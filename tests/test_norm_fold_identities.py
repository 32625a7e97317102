"""The identities behind the RMSNorm backward folded into the data-gradient
GEMMs, checked in fp64 on the oracle's own forward intermediates.

The backward of a block norm h = x r needs, per row, s = mean_j(dh_j h_j).
The bf16 step never forms dh for the two block norms; it takes the row sum
from quantities that the kernels before the norm's GEMM already hold:

* MLP norm: with u = h Wup^T, a = relu(u)^2, da the down-projection's input
  gradient and du = da 2 relu(u), dh = du Wup gives
  sum_j dh_j h_j = sum_f du_f u_f = 2 sum_f da_f a_f;
* attention norm: with qkv = h Wqkv^T the raw projection and dqkv its
  gradient, sum_j dh_j h_j = sum_c dqkv_c qkv_c, a sum of per-head shares;
  a value head's share is dv . v; a q or k head passes through RoPE (a
  rotation, which drops out of the dot product) and, with QK-norm,
  y = x r: its share is sum(dy y) eps r^2 (sum(dy y) without QK-norm);
* the update the folded epilogue applies, dx += r dh - (r s) h, equals the
  norm's backward r (dh - h mean(dh h)).

A slip in any of these (a lost factor 2, 1/F instead of 1/d, r^2 for eps r^2,
a head's share taken before the rotation, GQA heads miscounted) fails a test.
"""
import numpy as np
import pytest

import oracle
import synth
from oracle import gpt_oracle as go


def _cache(name="tiny", **kw):
    w = synth.workload(name, **kw)
    cfg = oracle.from_workload(w)
    params = {k: v.astype(np.float64) for k, v in synth.make_params(w).items()}
    tok, tgt = synth.make_tokens(w)
    cache = go.sequence_forward(cfg, params, tok[0], tgt[0])
    return w, cfg, params, cache


def _rng(seed):
    return np.random.default_rng(seed)


def test_mlp_row_sum_from_the_down_projection_gradient():
    w, cfg, params, cache = _cache()
    for l in range(cfg.n_layer):
        c = cache["layers"][l]
        wup, wdown = params[f"layers.{l}.wup"], params[f"layers.{l}.wdown"]
        dx = _rng(l).standard_normal(c["h2"].shape)          # gradient reaching the MLP output
        da = dx @ wdown
        du = da * 2.0 * np.maximum(c["u"], 0.0)
        dh = du @ wup
        lhs = np.sum(dh * c["h2"], axis=1)
        rhs = 2.0 * np.sum(da * c["a"], axis=1)
        scale = np.sum(np.abs(dh * c["h2"]), axis=1)
        assert np.all(np.abs(lhs - rhs) <= 1e-12 * scale), np.max(np.abs(lhs - rhs) / scale)
        # the folded update (s = (2/d) sum da a) is the norm's backward
        s = 2.0 * np.sum(da * c["a"], axis=1, keepdims=True) / w.d_model
        fold = c["r2"] * dh - (c["r2"] * s) * c["h2"]
        ref = go.rms_norm_backward(dh, c["h2"], c["r2"])
        np.testing.assert_allclose(fold, ref, rtol=1e-10, atol=1e-12 * np.max(np.abs(ref)))


@pytest.mark.parametrize("kw", [dict(norm_eps=0.1), dict(norm_eps=0.1, n_kv_head=2),
                                dict(qk_norm=False), dict(norm_eps=1e-6)])
def test_attention_row_sum_from_per_head_shares(kw):
    """eps = 0.1 makes the q/k shares (eps r^2 sum(dy y)) a visible part of the row sum."""
    w, cfg, params, cache = _cache(**kw)
    T, d, H, hd, Hkv = cache["tok"].shape[0], cfg.d_model, cfg.n_head, cfg.head_dim, cfg.kv_heads
    dkv = Hkv * hd
    cos, sin = cache["cos"], cache["sin"]
    for l in range(cfg.n_layer):
        c = cache["layers"][l]
        wqkv = params[f"layers.{l}.wqkv"]
        qkv = c["h"] @ wqkv.T                                  # the raw projection
        do = _rng(10 + l).standard_normal((T, H, hd))
        _, p, _ = go.causal_attention(c["qn"], c["kn"], c["v"], cfg.window)
        dqn, dkn, dv = go.causal_attention_backward(do, c["qn"], c["kn"], c["v"], p)
        if cfg.qk_norm:
            dq = go.rms_norm_backward(dqn, c["qn"], c["rq"])
            dk = go.rms_norm_backward(dkn, c["kn"], c["rk"])
        else:
            dq, dk = dqn, dkn
        dq = go.rope_backward(dq, cos, sin)
        dk = go.rope_backward(dk, cos, sin)
        dqkv = np.concatenate([dq.reshape(T, d), dk.reshape(T, dkv), dv.reshape(T, dkv)], axis=1)
        dh = dqkv @ wqkv
        total = np.sum(dh * c["h"], axis=1)
        scale = np.sum(np.abs(dh * c["h"]), axis=1) + np.sum(np.abs(dqkv * qkv), axis=1)
        assert np.all(np.abs(total - np.sum(dqkv * qkv, axis=1)) <= 1e-12 * scale)

        # each head's share as the attention kernels form it
        def share(dy, y, r):
            gy = np.sum(dy * y, axis=2)                         # [T, heads]
            return gy * cfg.norm_eps * r[..., 0] ** 2 if cfg.qk_norm else gy
        sq = share(dqn, c["qn"], c["rq"])
        sk = share(dkn, c["kn"], c["rk"])
        sv = np.sum(dv * qkv[:, d + dkv:].reshape(T, Hkv, hd), axis=2)
        # against the same dot products taken on the raw heads
        q_raw = qkv[:, :d].reshape(T, H, hd)
        k_raw = qkv[:, d:d + dkv].reshape(T, Hkv, hd)
        hscale = np.sum(np.abs(dqn * c["qn"]), axis=2)
        np.testing.assert_allclose(sq, np.sum(dq * q_raw, axis=2), rtol=1e-9, atol=1e-12 * np.max(hscale))
        np.testing.assert_allclose(sk, np.sum(dk * k_raw, axis=2), rtol=1e-9,
                                   atol=1e-12 * np.max(np.sum(np.abs(dkn * c["kn"]), axis=2)))
        parts = np.concatenate([sq, sk, sv], axis=1)            # [T, H + 2 Hkv], the kernels' layout
        assert parts.shape[1] == H + 2 * Hkv
        np.testing.assert_allclose(np.sum(parts, axis=1), total, rtol=1e-9, atol=1e-12 * np.max(scale))
        # the folded update with s = (1/d) sum of the shares
        s = np.sum(parts, axis=1, keepdims=True) / d
        fold = c["r1"] * dh - (c["r1"] * s) * c["h"]
        ref = go.rms_norm_backward(dh, c["h"], c["r1"])
        np.testing.assert_allclose(fold, ref, rtol=1e-9, atol=1e-12 * np.max(np.abs(ref)))


def test_qk_shares_vanish_with_eps_but_not_without_the_norm():
    """With QK-norm the q/k shares are eps r^2 sum(dy y): of order eps next to
    the value heads'; without it they are full-size dot products."""
    for kw, small in ((dict(norm_eps=1e-6), True), (dict(qk_norm=False), False)):
        w, cfg, params, cache = _cache(**kw)
        c = cache["layers"][0]
        T, H, hd = cache["tok"].shape[0], cfg.n_head, cfg.head_dim
        do = _rng(3).standard_normal((T, H, hd))
        _, p, _ = go.causal_attention(c["qn"], c["kn"], c["v"], cfg.window)
        dqn, _, dv = go.causal_attention_backward(do, c["qn"], c["kn"], c["v"], p)
        gy = np.sum(dqn * c["qn"], axis=2)
        sq = gy * cfg.norm_eps * c["rq"][..., 0] ** 2 if cfg.qk_norm else gy
        sv = np.sum(dv * c["v"], axis=2)
        ratio = np.max(np.abs(sq)) / np.max(np.abs(sv))
        assert (ratio < 1e-4) if small else (ratio > 1e-3), ratio
