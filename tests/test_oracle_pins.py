"""Pins for the fp64 CPU oracle: facts fixed by the mathematics, not by the oracle.

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a missing 1/N) breaks at least one:

* closed-form loss at initialisation (a missing final norm, a wrong mean);
* softmax rows summing to one, lower-triangular attention probabilities;
* causality: future tokens leave earlier logits and losses bit-identical;
* RoPE against cos/sin computed scalar by scalar, its relative-position
  property, norm preservation and the adjoint used by the backward;
* RMSNorm of a constant row;
* a two-token attention example and an L=0 (bigram) model, by hand with
  Python scalars;
* central finite differences of the whole step in fp64;
* an independent derivation of every gradient by torch autograd in float64,
  with torch's own RMSNorm, causal scaled-dot-product attention and
  cross-entropy in the forward.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth
from oracle import gpt_oracle as go

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small(name="tiny", **kw):
    w = synth.workload(name, **kw)
    return w, oracle.from_workload(w)


# ---------------------------------------------------------------------------
# loss at initialisation (closed form)
# ---------------------------------------------------------------------------

def _init_loss_check(w, res, tgt):
    """loss ~ ln V + sigma^2/2 with sigma^2 = 0.02^2 * d (hf has unit RMS).

    Given hf, the logits z_v = w_v . hf are iid N(0, sigma^2) over v, so
    E[logsumexp] = ln V + sigma^2/2 + O(1/V) and E[z_target] = 0.  Positions
    that share a target share w_v, so the spread of the mean scales with
    sqrt(sum_v q_v^2), q_v the empirical target frequency.
    """
    sig2 = 0.02 ** 2 * w.d_model
    expect = math.log(w.vocab) + sig2 / 2
    q = np.bincount(tgt.ravel(), minlength=w.vocab) / tgt.size
    bound = 0.02 + 4 * math.sqrt(sig2) * math.sqrt(float(np.sum(q * q)))
    assert abs(res.loss - expect) <= bound, (res.loss, expect, bound)


def test_loss_at_init_tiny():
    w, cfg = small()
    tok, tgt = synth.make_tokens(w)
    res = oracle.step(cfg, synth.make_params(w), tok, tgt, backward=False)
    _init_loss_check(w, res, tgt)


def test_loss_at_init_wide_vocab():
    # story-model width and vocabulary, shortened so it runs in a second
    w, cfg = small("story", n_layer=1, seq_len=64, batch=4)
    tok, tgt = synth.make_tokens(w)
    res = oracle.step(cfg, synth.make_params(w), tok, tgt, backward=False)
    _init_loss_check(w, res, tgt)


def test_golden_loss_table_matches_closed_form():
    with open(os.path.join(GOLDEN, "loss_at_init.json")) as f:
        table = json.load(f)
    for name, row in table["workloads"].items():
        w = synth.workload(name)
        assert row["vocab"] == w.vocab and row["d_model"] == w.d_model
        assert abs(row["expected_loss"] - (math.log(w.vocab) + 0.02 ** 2 * w.d_model / 2)) < 5e-4


def test_uniform_logits_give_log_v():
    z = np.zeros((3, 17))
    loss, lse, p = go.cross_entropy(z, np.array([0, 5, 16]))
    assert np.allclose(loss, math.log(17), rtol=0, atol=1e-14)
    assert np.allclose(p, 1 / 17, atol=1e-16)


# ---------------------------------------------------------------------------
# softmax / attention structure
# ---------------------------------------------------------------------------

def test_softmax_rows_sum_to_one_and_causal_structure():
    w, cfg = small()
    tok, tgt = synth.make_tokens(w)
    res = oracle.step(cfg, synth.make_params(w), tok, tgt, backward=False, keep_caches=True)
    c = res.caches[0]
    assert np.max(np.abs(c["probs"].sum(-1) - 1)) <= 1e-12
    assert np.all(c["lse_z"] >= c["z"].max(-1))
    for lay in c["layers"]:
        _, p, lse = go.causal_attention(lay["qn"], lay["kn"], lay["v"])
        assert np.max(np.abs(p.sum(-1) - 1)) <= 1e-12
        assert np.all(np.triu(p, k=1) == 0.0)      # nothing from the future
        assert np.all(p >= 0)


def test_attention_single_position_returns_v():
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((1, 3, 8)) for _ in range(3))
    o, p, lse = go.causal_attention(q, k, v)
    assert np.array_equal(o, v)
    assert np.allclose(lse, (q * k).sum(-1).T / math.sqrt(8), atol=1e-15)


def test_attention_two_positions_by_hand():
    q = np.array([[[1.0, 0.0]], [[0.5, -1.0]]])     # [T=2, H=1, hd=2]
    k = np.array([[[2.0, 1.0]], [[0.0, 3.0]]])
    v = np.array([[[1.0, 2.0]], [[-1.0, 4.0]]])
    o, _, _ = go.causal_attention(q, k, v)
    assert np.allclose(o[0, 0], [1.0, 2.0], atol=1e-15)
    s0 = (0.5 * 2.0 + -1.0 * 1.0) / math.sqrt(2)
    s1 = (0.5 * 0.0 + -1.0 * 3.0) / math.sqrt(2)
    e0, e1 = math.exp(s0), math.exp(s1)
    p0, p1 = e0 / (e0 + e1), e1 / (e0 + e1)
    assert np.allclose(o[1, 0], [p0 * 1.0 + p1 * -1.0, p0 * 2.0 + p1 * 4.0], atol=1e-14)


# ---------------------------------------------------------------------------
# causality of the whole model
# ---------------------------------------------------------------------------

def test_future_tokens_leave_past_bit_identical():
    w, cfg = small()
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    a = oracle.step(cfg, params, tok, tgt, backward=False, keep_caches=True)
    tok2 = tok.copy()
    b, t = 1, 20
    rng = np.random.default_rng(1)
    tok2[b, t + 1:] = rng.integers(0, w.vocab, size=w.seq_len - t - 1)
    assert not np.array_equal(tok, tok2)
    r = oracle.step(cfg, params, tok2, tgt, backward=False, keep_caches=True)
    assert np.array_equal(a.caches[b]["z"][: t + 1], r.caches[b]["z"][: t + 1])
    assert np.array_equal(a.token_loss[b, : t + 1], r.token_loss[b, : t + 1])
    assert not np.array_equal(a.token_loss[b, t + 1:], r.token_loss[b, t + 1:])
    for other in range(w.batch):
        if other != b:
            assert np.array_equal(a.token_loss[other], r.token_loss[other])


# ---------------------------------------------------------------------------
# RoPE and RMSNorm special cases
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("hd", [4, 16, 128])
def test_rope_basis_vectors_match_scalar_cos_sin(hd):
    T = 9
    base = 10000.0
    cos, sin = go.rope_tables(T, hd, base)
    half = hd // 2
    for i in [0, half // 2, half - 1]:
        e = np.zeros((T, 1, hd))
        e[:, 0, i] = 1.0
        y = go.rope(e, cos, sin)
        for t in range(T):
            ang = t * base ** (-2.0 * i / hd)
            want = np.zeros(hd)
            want[i] = math.cos(ang)
            want[i + half] = math.sin(ang)
            assert np.allclose(y[t, 0], want, atol=1e-15)


def test_rope_identity_at_zero_norm_preserving_and_relative():
    rng = np.random.default_rng(3)
    T, H, hd = 12, 2, 16
    cos, sin = go.rope_tables(T, hd, 10000.0)
    x = rng.standard_normal((T, H, hd))
    y = go.rope(x, cos, sin)
    assert np.array_equal(y[0], x[0])
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-14)
    q = np.repeat(rng.standard_normal((1, 1, hd)), T, axis=0)
    k = np.repeat(rng.standard_normal((1, 1, hd)), T, axis=0)
    rq, rk = go.rope(q, cos, sin), go.rope(k, cos, sin)
    # <R(t1) q, R(t2) k> depends on t1 - t2 only
    for shift in range(1, 4):
        assert np.allclose(rq[5, 0] @ rk[2, 0], rq[5 + shift, 0] @ rk[2 + shift, 0], atol=1e-13)
    # the backward is the adjoint of the forward rotation
    g = rng.standard_normal((T, H, hd))
    assert np.isclose(np.sum(y * g), np.sum(x * go.rope_backward(g, cos, sin)), rtol=1e-13)


def test_rms_norm_constant_row():
    for c in [3.0, -0.25, 1e-3]:
        x = np.full((1, 64), c)
        y, r = go.rms_norm(x, 1e-6)
        want = c / math.sqrt(c * c + 1e-6)
        assert np.allclose(y, want, rtol=1e-15)
        assert np.isclose(r[0, 0], 1 / math.sqrt(c * c + 1e-6), rtol=1e-15)


def test_bigram_model_by_hand():
    # L = 0: z = rms(wte[tok]) . lm_head^T; worked with Python scalars
    w, cfg = small("tiny", n_layer=0, d_model=2, n_head=1, head_dim=2, vocab=2, seq_len=1, batch=1)
    params = {"wte": np.array([[3.0, 4.0], [1.0, -1.0]]),
              "lm_head": np.array([[0.5, -1.0], [2.0, 0.25]])}
    tok, tgt = np.array([[0]]), np.array([[1]])
    res = oracle.step(cfg, params, tok, tgt)
    m = (9.0 + 16.0) / 2
    r = 1 / math.sqrt(m + 1e-6)
    h = [3.0 * r, 4.0 * r]
    z = [0.5 * h[0] - 1.0 * h[1], 2.0 * h[0] + 0.25 * h[1]]
    lse = math.log(math.exp(z[0]) + math.exp(z[1]))
    assert math.isclose(res.loss, lse - z[1], rel_tol=1e-14)
    p = [math.exp(z[0] - lse), math.exp(z[1] - lse)]
    g = [p[0], p[1] - 1.0]
    want_dlm = np.array([[g[0] * h[0], g[0] * h[1]], [g[1] * h[0], g[1] * h[1]]])
    assert np.allclose(res.grads["lm_head"], want_dlm, rtol=1e-13)
    # d/dx of rms(x) along the 2-vector, composed with dz/dh = lm_head^T g
    dh = [g[0] * 0.5 + g[1] * 2.0, g[0] * -1.0 + g[1] * 0.25]
    dot = (dh[0] * h[0] + dh[1] * h[1]) / 2
    dx = [r * (dh[0] - h[0] * dot), r * (dh[1] - h[1] * dot)]
    assert np.allclose(res.grads["wte"][0], dx, rtol=1e-12)
    assert np.array_equal(res.grads["wte"][1], [0.0, 0.0])


# ---------------------------------------------------------------------------
# finite differences
# ---------------------------------------------------------------------------

def test_central_finite_differences_tiny():
    w, cfg = small("tiny", batch=2)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    res = oracle.step(cfg, params, tok, tgt)
    rng = np.random.default_rng(7)
    worst = 0.0
    for name, p in params.items():
        if name == "wte":
            rows = np.unique(tok)
            coords = [(int(rng.choice(rows)), int(rng.integers(p.shape[1]))) for _ in range(16)]
        else:
            coords = [(int(rng.integers(p.shape[0])), int(rng.integers(p.shape[1]))) for _ in range(16)]
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
            worst = max(worst, err)
            assert err <= 1e-5, (name, i, j, fd, res.grads[name][i, j])
    assert worst < 1e-5


# ---------------------------------------------------------------------------
# independent autograd derivation (torch, float64, CPU)
# ---------------------------------------------------------------------------

def _torch_step(w, params, tok, tgt):
    import torch
    import torch.nn.functional as F

    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in params.items()}
    B, T = tok.shape
    d, H, hd = w.d_model, w.n_head, w.head_dim
    i = torch.arange(hd // 2, dtype=torch.float64)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * (w.rope_base ** (-2.0 * i / hd))[None]
    cos, sin = torch.cos(ang)[None, :, None, :], torch.sin(ang)[None, :, None, :]

    def rot(x):
        a, b = x[..., : hd // 2], x[..., hd // 2:]
        return torch.cat([a * cos - b * sin, a * sin + b * cos], -1)

    def norm(x):
        return F.rms_norm(x, (x.shape[-1],), eps=w.norm_eps)

    x = t["wte"][torch.tensor(tok, dtype=torch.long)]
    for l in range(w.n_layer):
        qkv = F.linear(norm(x), t[f"layers.{l}.wqkv"])
        q, k, v = qkv.split(d, dim=-1)
        q = norm(rot(q.view(B, T, H, hd)))
        k = norm(rot(k.view(B, T, H, hd)))
        v = v.view(B, T, H, hd)
        o = F.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2),
                                           is_causal=True)
        x = x + F.linear(o.transpose(1, 2).reshape(B, T, d), t[f"layers.{l}.wo"])
        u = F.linear(norm(x), t[f"layers.{l}.wup"])
        x = x + F.linear(torch.relu(u).square(), t[f"layers.{l}.wdown"])
    z = F.linear(norm(x), t["lm_head"])
    loss = F.cross_entropy(z.view(B * T, -1), torch.tensor(tgt, dtype=torch.long).view(-1))
    loss.backward()
    return float(loss), {k: v.grad.numpy() for k, v in t.items()}


@pytest.mark.parametrize("name,kw", [("tiny", {}),
                                     ("story", dict(n_layer=2, seq_len=48, batch=2, vocab=512))])
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


def test_rows_subset_reassembles_full_step():
    w, cfg = small()
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    full = oracle.step(cfg, params, tok, tgt)
    parts = [oracle.step(cfg, params, tok, tgt, rows=[b]) for b in range(w.batch)]
    assert np.allclose(sum(p.loss for p in parts), full.loss, rtol=1e-14)
    for k in params:
        assert np.allclose(sum(p.grads[k] for p in parts), full.grads[k], rtol=1e-12, atol=1e-18)
