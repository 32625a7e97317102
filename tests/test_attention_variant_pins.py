"""Pins for the oracle's grouped-query (GQA) and sliding-window attention.

Facts fixed by the definitions, not by the oracle's code:

* GQA with key/value heads shared by groups of query heads is multi-head
  attention whose key/value projection rows are repeated per query head: the
  same loss, the same query and MLP gradients, and a shared head's gradient
  equal to the sum of its copies' gradients;
* a window at least as long as the sequence is the full causal window, bit for
  bit;
* a window of one position attends to the query position alone (o = v);
* the receptive field of L layers with window W is the L(W-1) previous
  positions: a token further back leaves the logits bit-identical, the token
  exactly that far back does not;
* central finite differences of the whole step, and torch autograd in float64
  with torch's own grouped-query scaled-dot-product attention and an explicit
  window mask.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from oracle import gpt_oracle as go


def small(name="tiny", **kw):
    w = synth.workload(name, **kw)
    return w, oracle.from_workload(w)


def _mha_params(w, params):
    """The multi-head model equal to the GQA model `w`: each key/value head's
    W_qkv rows repeated once per query head that reads it."""
    d, H, hd, Hkv = w.d_model, w.n_head, w.head_dim, w.n_kv_head
    rep = H // Hkv
    out = dict(params)
    for l in range(w.n_layer):
        wqkv = params[f"layers.{l}.wqkv"]
        q, k, v = wqkv[:d], wqkv[d:d + Hkv * hd], wqkv[d + Hkv * hd:]
        heads = lambda m: [m[(h // rep) * hd:(h // rep + 1) * hd] for h in range(H)]
        out[f"layers.{l}.wqkv"] = np.concatenate([q] + heads(k) + heads(v), axis=0)
    return out


@pytest.mark.parametrize("n_kv_head,window", [(2, 0), (1, 0), (2, 6)])
def test_gqa_equals_mha_with_repeated_kv_rows(n_kv_head, window):
    w, cfg = small("tiny", n_kv_head=n_kv_head, window=window, batch=2, seq_len=24)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    g = oracle.step(cfg, params, tok, tgt)
    wm = w.replace(n_kv_head=0)
    m = oracle.step(oracle.from_workload(wm), _mha_params(w, params), tok, tgt)
    assert math.isclose(g.loss, m.loss, rel_tol=1e-13)
    d, H, hd = w.d_model, w.n_head, w.head_dim
    rep = H // n_kv_head
    for name in params:
        if not name.endswith(".wqkv"):
            assert np.allclose(g.grads[name], m.grads[name], rtol=1e-10, atol=1e-16), name
            continue
        gg, mg = g.grads[name], m.grads[name]
        assert np.allclose(gg[:d], mg[:d], rtol=1e-10, atol=1e-16)
        for part in range(2):  # k, then v
            for kh in range(n_kv_head):
                got = gg[d + (part * n_kv_head + kh) * hd:][:hd]
                want = sum(mg[d + (part * H + h) * hd:][:hd] for h in range(kh * rep, (kh + 1) * rep))
                assert np.allclose(got, want, rtol=1e-10, atol=1e-16), (name, part, kh)


def test_window_covering_the_sequence_is_full_causal():
    w, cfg = small("tiny", batch=2, seq_len=20)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    full = oracle.step(cfg, params, tok, tgt)
    for W in (20, 33):
        r = oracle.step(oracle.from_workload(w.replace(window=W)), params, tok, tgt)
        assert r.loss == full.loss
        for k in params:
            assert np.array_equal(r.grads[k], full.grads[k]), (W, k)


def test_window_of_one_returns_v():
    rng = np.random.default_rng(11)
    T, H, Hkv, hd = 9, 4, 2, 8
    q = rng.standard_normal((T, H, hd))
    k, v = rng.standard_normal((T, Hkv, hd)), rng.standard_normal((T, Hkv, hd))
    o, p, lse = go.causal_attention(q, k, v, window=1)
    for h in range(H):
        assert np.array_equal(o[:, h], v[:, h // (H // Hkv)])
    assert np.array_equal(p, np.broadcast_to(np.eye(T), p.shape))
    # lse of a single score is that score
    s = np.einsum("thd,thd->ht", q, np.repeat(k, H // Hkv, axis=1)) / math.sqrt(hd)
    assert np.allclose(lse, s, rtol=1e-15, atol=1e-15)


def test_mask_counts():
    for T, W in [(10, 3), (7, 1), (5, 9)]:
        m = go.attention_mask(T, W)
        # row i sees min(i + 1, W) keys, all at or before i
        assert list(m.sum(1)) == [min(i + 1, W) for i in range(T)]
        assert not np.any(np.triu(m, k=1))


@pytest.mark.parametrize("n_layer,window", [(1, 5), (2, 4)])
def test_window_receptive_field(n_layer, window):
    w, cfg = small("tiny", n_layer=n_layer, window=window, n_kv_head=2, batch=1, seq_len=32)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    base = oracle.step(cfg, params, tok, tgt, backward=False, keep_caches=True)
    i = 30
    reach = n_layer * (window - 1)
    far = tok.copy()
    far[0, i - reach - 1] = (far[0, i - reach - 1] + 1) % w.vocab
    r = oracle.step(cfg, params, far, tgt, backward=False, keep_caches=True)
    assert np.array_equal(base.caches[0]["z"][i], r.caches[0]["z"][i])
    near = tok.copy()
    near[0, i - reach] = (near[0, i - reach] + 1) % w.vocab
    r = oracle.step(cfg, params, near, tgt, backward=False, keep_caches=True)
    assert not np.array_equal(base.caches[0]["z"][i], r.caches[0]["z"][i])


def test_central_finite_differences_gqa_window():
    w, cfg = small("tiny", n_kv_head=2, window=5, batch=2, seq_len=16)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    res = oracle.step(cfg, params, tok, tgt)
    rng = np.random.default_rng(13)
    d, hd = w.d_model, w.head_dim
    for name, p in params.items():
        if name == "wte":
            rows = np.unique(tok)
            coords = [(int(rng.choice(rows)), int(rng.integers(p.shape[1]))) for _ in range(8)]
        elif name.endswith(".wqkv"):
            # rows of every part: q, the first and second k head, v
            picks = [d // 2, d + 1, d + hd + 3, d + 2 * hd + 5, d + 3 * hd + 7]
            coords = [(r, int(rng.integers(p.shape[1]))) for r in picks for _ in range(2)]
        else:
            coords = [(int(rng.integers(p.shape[0])), int(rng.integers(p.shape[1]))) for _ in range(8)]
        gscale = np.max(np.abs(res.grads[name]))
        for (i, j) in coords:
            h = 1e-5 * max(1.0, abs(p[i, j]))
            saved = p[i, j]
            p[i, j] = saved + h
            lp = oracle.step(cfg, params, tok, tgt, backward=False).loss
            p[i, j] = saved - h
            lm = oracle.step(cfg, params, tok, tgt, backward=False).loss
            p[i, j] = saved
            fd = (lp - lm) / (2 * h)
            err = abs(fd - res.grads[name][i, j]) / max(abs(res.grads[name][i, j]), 1e-3 * gscale)
            assert err <= 1e-5, (name, i, j, fd, res.grads[name][i, j])


def _torch_step(w, params, tok, tgt):
    """The step in torch float64 with torch's own GQA attention (enable_gqa)
    and the window as an explicit boolean mask."""
    import torch
    import torch.nn.functional as F

    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in params.items()}
    B, T = tok.shape
    d, H, hd, Hkv = w.d_model, w.n_head, w.head_dim, w.n_kv_head or w.n_head
    i = torch.arange(hd // 2, dtype=torch.float64)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * (w.rope_base ** (-2.0 * i / hd))[None]
    cos, sin = torch.cos(ang)[None, :, None, :], torch.sin(ang)[None, :, None, :]
    pos = torch.arange(T)
    mask = pos[None, :] <= pos[:, None]
    if w.window:
        mask &= (pos[:, None] - pos[None, :]) < w.window

    def rot(x):
        a, b = x[..., : hd // 2], x[..., hd // 2:]
        return torch.cat([a * cos - b * sin, a * sin + b * cos], -1)

    def norm(x):
        return F.rms_norm(x, (x.shape[-1],), eps=w.norm_eps)

    x = t["wte"][torch.tensor(tok, dtype=torch.long)]
    for l in range(w.n_layer):
        qkv = F.linear(norm(x), t[f"layers.{l}.wqkv"])
        q, k, v = qkv.split([d, Hkv * hd, Hkv * hd], dim=-1)
        q = norm(rot(q.view(B, T, H, hd)))
        k = norm(rot(k.view(B, T, Hkv, hd)))
        v = v.view(B, T, Hkv, hd)
        o = F.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2),
                                           attn_mask=mask, enable_gqa=True)
        x = x + F.linear(o.transpose(1, 2).reshape(B, T, d), t[f"layers.{l}.wo"])
        u = F.linear(norm(x), t[f"layers.{l}.wup"])
        x = x + F.linear(torch.relu(u).square(), t[f"layers.{l}.wdown"])
    z = F.linear(norm(x), t["lm_head"])
    loss = F.cross_entropy(z.view(B * T, -1), torch.tensor(tgt, dtype=torch.long).view(-1))
    loss.backward()
    return float(loss), {k: v.grad.numpy() for k, v in t.items()}


@pytest.mark.parametrize("name,kw", [
    ("tiny", dict(n_kv_head=2, window=7)),
    ("tiny", dict(n_kv_head=1, window=0)),
    ("story", dict(n_layer=2, seq_len=48, batch=2, vocab=512, n_kv_head=2, window=20)),
])
def test_backward_matches_torch_autograd_f64(name, kw):
    w, cfg = small(name, **kw)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    res = oracle.step(cfg, params, tok, tgt)
    tl, tg = _torch_step(w, params, tok, tgt)
    assert math.isclose(res.loss, tl, rel_tol=1e-12)
    for k in params:
        ref = tg[k]
        err = np.max(np.abs(res.grads[k] - ref)) / np.max(np.abs(ref))
        assert err <= 1e-10, (k, err)
