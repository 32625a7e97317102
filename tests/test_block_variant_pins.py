"""Pins of the oracle's block variants ("ChatGPT'nizi 50 Dolara Nasil
Egitirsiniz?", section "1. GPT Modeli": the value-embedding (ResFormer) and
efficiency-trick listings): value embeddings with a per-head gate, per-layer
residual scaling, smear and backout.

* neutral values (residual scales (1, 0), smear and backout scales 0, zero
  value embeddings) give the plain model's loss and gradients bit for bit;
* smear mixes exactly the previous position: with no layers, position t's
  loss depends on tokens t and t-1 only, and position 0 on token 0 only;
* causality still holds: later tokens leave earlier losses bit-identical;
* the backout point and x0 are where the readings put them (a model whose
  stream is changed only there moves by the predicted amount);
* central finite differences of the whole step on every variant parameter;
* torch float64 autograd of an independently written forward (torch's own
  RMSNorm, attention with enable_gqa, sigmoid and cross-entropy) agrees to
  1e-10.
"""
import math

import numpy as np
import pytest

import oracle
import synth

ALL = dict(ve_every=1, resid_lambdas=True, smear=True, backout=True)


def small(name="tiny", **kw):
    w = synth.workload(name, **kw)
    return w, oracle.from_workload(w)


def test_neutral_values_give_the_plain_model_bit_for_bit():
    w, cfg = small("tiny", n_kv_head=2, batch=2, seq_len=20, **ALL)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    params["lambdas"][:] = [1.0, 0.0]
    params["scalars"][:] = 0.0
    for l in range(w.n_layer):
        params[f"ve.{l}"][:] = 0.0
    res = oracle.step(cfg, params, tok, tgt)
    wp = w.replace(ve_every=0, resid_lambdas=False, smear=False, backout=False)
    plain = oracle.step(oracle.from_workload(wp), {k: params[k] for k, _ in synth.param_shapes(wp)},
                        tok, tgt)
    assert res.loss == plain.loss
    for k in plain.grads:
        assert np.array_equal(res.grads[k], plain.grads[k]), k


def test_smear_reaches_exactly_one_position_back():
    w, cfg = small("tiny", n_layer=0, batch=1, seq_len=12, smear=True)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    base = oracle.step(cfg, params, tok, tgt, backward=False).token_loss[0]
    t = 7
    for back, moves in ((1, True), (2, False), (5, False)):
        tok2 = tok.copy()
        tok2[0, t - back] = (tok2[0, t - back] + 1) % w.vocab
        got = oracle.step(cfg, params, tok2, tgt, backward=False).token_loss[0]
        assert (got[t] != base[t]) == moves, back
    # position 0 has no previous token: its loss is the plain bigram model's
    wp = w.replace(smear=False)
    plain = oracle.step(oracle.from_workload(wp), {k: params[k] for k, _ in synth.param_shapes(wp)},
                        tok, tgt, backward=False).token_loss[0]
    assert base[0] == plain[0] and base[1] != plain[1]


def test_causality_with_every_variant():
    w, cfg = small("tiny", batch=1, seq_len=16, **ALL)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    base = oracle.step(cfg, params, tok, tgt, backward=False).token_loss[0]
    tok2 = tok.copy()
    tok2[0, 9:] = (tok2[0, 9:] + 3) % w.vocab
    got = oracle.step(cfg, params, tok2, tgt, backward=False).token_loss[0]
    assert np.array_equal(got[:9], base[:9]) and not np.array_equal(got[9:], base[9:])


def test_backout_and_x0_placement():
    # with every block's output projection zero, the stream never changes after
    # the embedding: x_L = x_b = x0 = e, so backout leaves (1 - beta) e and the
    # residual scales multiply e by prod(a_l + b_l)
    w, cfg = small("tiny", batch=1, seq_len=10, resid_lambdas=True, backout=True)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    for l in range(w.n_layer):
        params[f"layers.{l}.wo"][:] = 0.0
        params[f"layers.{l}.wdown"][:] = 0.0
    params["lambdas"][:] = [[1.25, 0.5], [0.8, -0.2]]
    params["scalars"][0, 1] = 0.75
    cache = oracle.gpt_oracle.sequence_forward(cfg, params, tok[0], tgt[0])
    e = params["wte"][tok[0]]
    # layer 0: 1.75 e; layer 1 (the backout layer, n_layer // 2): 0.8*1.75 e - 0.2 e = 1.2 e
    assert np.allclose(cache["x_b"], 1.2 * e, rtol=1e-14)
    assert np.allclose(cache["x_out"], (1.0 - 0.75) * 1.2 * e, rtol=1e-13)
    assert np.array_equal(cache["x0"], e)


def test_central_finite_differences_every_variant():
    w, cfg = small("tiny", n_kv_head=2, batch=2, seq_len=12, ve_gate_channels=16, **ALL)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    res = oracle.step(cfg, params, tok, tgt)
    rng = np.random.default_rng(31)
    names = ["wte", "layers.0.wqkv", "layers.1.wup", "lm_head", "ve.0", "ve.1", "ve_gate.0",
             "ve_gate.1", "lambdas", "smear_gate", "scalars"]
    for name in names:
        p = params[name]
        if name in ("wte", "ve.0", "ve.1"):
            rows = np.unique(tok)
            coords = [(int(rng.choice(rows)), int(rng.integers(p.shape[1]))) for _ in range(6)]
        elif name in ("lambdas", "scalars"):
            coords = [(i, j) for i in range(p.shape[0]) for j in range(p.shape[1])]
        else:
            coords = [(int(rng.integers(p.shape[0])), int(rng.integers(p.shape[1]))) for _ in range(6)]
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
    """The step in torch float64, written from the readings independently of
    the oracle, differentiated by autograd."""
    import torch
    import torch.nn.functional as F

    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in params.items()}
    B, T = tok.shape
    d, H, hd, Hkv = w.d_model, w.n_head, w.head_dim, w.n_kv_head or w.n_head
    i = torch.arange(hd // 2, dtype=torch.float64)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * (w.rope_base ** (-2.0 * i / hd))[None]
    cos, sin = torch.cos(ang)[None, :, None, :], torch.sin(ang)[None, :, None, :]
    ids = torch.tensor(tok, dtype=torch.long)

    def rot(x):
        a, b = x[..., : hd // 2], x[..., hd // 2:]
        return torch.cat([a * cos - b * sin, a * sin + b * cos], -1)

    def norm(x):
        return F.rms_norm(x, (x.shape[-1],), eps=w.norm_eps)

    x = t["wte"][ids]
    if w.smear:
        g = t["scalars"][0, 0] * torch.sigmoid(F.linear(x[:, :, :24], t["smear_gate"]))  # [B, T, 1]
        x = x + g * F.pad(x, (0, 0, 1, 0))[:, :-1]
    x0 = x
    xb = None
    for l in range(w.n_layer):
        if w.resid_lambdas:
            x = t["lambdas"][l, 0] * x + t["lambdas"][l, 1] * x0
        if w.backout and l == w.n_layer // 2:
            xb = x
        h = norm(x)
        qkv = F.linear(h, t[f"layers.{l}.wqkv"])
        q, k, v = qkv.split([d, Hkv * hd, Hkv * hd], dim=-1)
        v = v.view(B, T, Hkv, hd)
        if w.ve_every and l % w.ve_every == w.ve_every - 1:
            gate = 3 * torch.sigmoid(F.linear(h[..., :w.ve_gate_channels], t[f"ve_gate.{l}"]))
            v = v + gate.unsqueeze(-1) * t[f"ve.{l}"][ids].view(B, T, Hkv, hd)
        q = norm(rot(q.view(B, T, H, hd)))
        k = norm(rot(k.view(B, T, Hkv, hd)))
        o = F.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2),
                                           is_causal=True, enable_gqa=True)
        x = x + F.linear(o.transpose(1, 2).reshape(B, T, d), t[f"layers.{l}.wo"])
        u = F.linear(norm(x), t[f"layers.{l}.wup"])
        x = x + F.linear(torch.relu(u).square(), t[f"layers.{l}.wdown"])
    if w.backout:
        x = x - t["scalars"][0, 1] * xb
    z = F.linear(norm(x), t["lm_head"])
    loss = F.cross_entropy(z.view(B * T, -1), torch.tensor(tgt, dtype=torch.long).view(-1))
    loss.backward()
    return float(loss.detach()), {k: v.grad.numpy() for k, v in t.items()}


@pytest.mark.parametrize("name,kw", [
    ("tiny", ALL),
    ("tiny", dict(n_kv_head=1, ve_every=2, ve_gate_channels=8, smear=True)),
    ("tiny", dict(n_layer=3, resid_lambdas=True, backout=True)),
    ("story", dict(n_layer=2, seq_len=40, batch=2, vocab=512, n_kv_head=2, **ALL)),
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
