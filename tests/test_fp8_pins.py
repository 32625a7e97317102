"""Pins for the oracle's FP8 (e4m3) block projections: forward and data gradient.

Facts fixed outside the oracle's code:

* the e4m3 value table and round-to-nearest-even against torch's own
  float8_e4m3fn conversion (a library routine), ties and subnormals included;
* the power-of-two scale: amax * 2^k <= 448 < amax * 2^(k+1);
* operands already on the scaled e4m3 grid pass through exactly;
* the product's error stays inside the bound two e4m3 roundings allow;
* the data gradient dY W with dY through e4m3 per row: exact for operands on
  the grid, inside the two-rounding bound otherwise;
* the whole step (multi-head, and grouped-query with a window) against torch
  float64 autograd in which each block projection quantizes through torch's
  bf16 and float8 casts with a log2-derived exponent, its backward written as
  its own autograd function (dY through the same casts for dX = dY W, the
  unquantized dY and X for dW).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import gpt_oracle as go


def test_e4m3_table_matches_torch_decode():
    vals, codes = go._e4m3_table()
    t = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    assert np.array_equal(vals, t.numpy())
    assert vals[-1] == 448.0 and vals[1] == 2.0 ** -9


def test_e4m3_round_matches_torch_cast():
    rng = np.random.default_rng(21)
    vals, _ = go._e4m3_table()
    mids = (vals[1:] + vals[:-1]) / 2                       # exact ties
    x = np.concatenate([
        rng.standard_normal(20000) * np.exp2(rng.integers(-12, 8, 20000)),
        mids, -mids, vals, rng.uniform(0, 2.0 ** -6, 2000)])  # subnormal range
    x = np.clip(x, -448, 448)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(go.e4m3_round(x), want)


def test_pow2_exponent_is_the_largest_fitting_power():
    rng = np.random.default_rng(3)
    amax = np.concatenate([rng.uniform(0.1, 10, 500) * np.exp2(rng.integers(-40, 20, 500)),
                           448.0 * np.exp2(np.arange(-10, 10.0)), [0.0]])
    k = go.pow2_exponent(amax)
    pos = amax > 0
    assert np.all(np.ldexp(amax[pos], k[pos]) <= 448)
    assert np.all(np.ldexp(amax[pos], k[pos] + 1) > 448)
    assert k[-1] == 0
    assert list(k[500:520]) == list(range(10, -10, -1))   # amax = 448 * 2^j -> k = -j


def test_fp8_linear_exact_on_grid():
    rng = np.random.default_rng(5)
    vals, _ = go._e4m3_table()
    grid = np.concatenate([vals, -vals])
    x = rng.choice(grid, (6, 32))
    x[:, 0] = 448.0                                  # row amax 448 * 2^-3 after scaling
    x = x * 2.0 ** -3
    w = rng.choice(grid, (5, 32))
    w[0, 0] = -448.0
    w = w * 2.0 ** 5
    assert np.array_equal(go.fp8_linear(x, w), x @ w.T)


def test_fp8_linear_error_bound():
    rng = np.random.default_rng(9)
    x = go._round_bf16(rng.standard_normal((16, 256)))
    w = go._round_bf16(rng.standard_normal((24, 256)) * 0.02)
    got = go.fp8_linear(x, w)
    exact = x @ w.T
    # each operand: relative error <= 2^-4 (3 mantissa bits, round to nearest),
    # or absolute <= 2^-10 (subnormal spacing 2^-9) in scaled units
    kx = go.pow2_exponent(np.abs(x).max(1))[:, None]
    kw = go.pow2_exponent(np.abs(w).max())
    ex = np.maximum(np.abs(x) * 2.0 ** -4, np.ldexp(2.0 ** -10, -kx))
    ew = np.maximum(np.abs(w) * 2.0 ** -4, np.ldexp(2.0 ** -10, -kw))
    bound = np.abs(x) @ ew.T + ex @ np.abs(w).T + ex @ ew.T
    assert np.all(np.abs(got - exact) <= bound * (1 + 1e-12))
    assert np.abs(got - exact).max() > 0


def test_fp8_dgrad_exact_on_grid():
    rng = np.random.default_rng(15)
    vals, _ = go._e4m3_table()
    grid = np.concatenate([vals, -vals])
    dy = rng.choice(grid, (7, 24))
    dy[:, 3] = -448.0                                 # row amax 448 * 2^-11 after scaling
    dy = dy * 2.0 ** -11
    w = rng.choice(grid, (24, 40))
    w[5, 1] = 448.0
    w = w * 2.0 ** 2
    assert np.array_equal(go._dgrad(dy, w, go.fp8_tensor(w)), dy @ w)
    assert np.array_equal(go._dgrad(dy, w, None), dy @ w)


def test_fp8_dgrad_error_bound():
    rng = np.random.default_rng(17)
    dy = go._round_bf16(rng.standard_normal((12, 200)) * 1e-4)
    w = go._round_bf16(rng.standard_normal((200, 96)) * 0.02)
    got = go._dgrad(dy, w, go.fp8_tensor(w))
    exact = dy @ w
    ky = go.pow2_exponent(np.abs(dy).max(1))[:, None]
    kw = go.pow2_exponent(np.abs(w).max())
    ey = np.maximum(np.abs(dy) * 2.0 ** -4, np.ldexp(2.0 ** -10, -ky))
    ew = np.maximum(np.abs(w) * 2.0 ** -4, np.ldexp(2.0 ** -10, -kw))
    bound = np.abs(dy) @ ew + ey @ np.abs(w) + ey @ ew
    assert np.all(np.abs(got - exact) <= bound * (1 + 1e-12))
    assert np.abs(got - exact).max() > 0


def _torch_fp8_step(w, params, tok, tgt):
    import torch.nn.functional as F

    def q(x):
        """x (float64) -> bf16 -> scaled e4m3 -> float64 value, via torch casts."""
        xb = x.to(torch.bfloat16).to(torch.float64)
        amax = xb.abs().amax(dim=-1, keepdim=True)
        k = torch.floor(torch.log2(448.0 / torch.where(amax > 0, amax, torch.ones_like(amax))))
        k = torch.where(torch.ldexp(amax, k) > 448, k - 1, k)
        k = torch.where(torch.ldexp(amax, k + 1) <= 448, k + 1, k)
        k = torch.where(amax > 0, k, torch.zeros_like(k))
        return torch.ldexp(torch.ldexp(xb, k).to(torch.float8_e4m3fn).to(torch.float64), -k)

    class Fp8Linear(torch.autograd.Function):
        @staticmethod
        def forward(ctx, x, W):
            xq = q(x.reshape(-1, x.shape[-1])).reshape(x.shape)
            wq = q(W.reshape(1, -1)).reshape(W.shape)          # one scale per tensor
            ctx.save_for_backward(x, wq)
            return xq @ wq.T

        @staticmethod
        def backward(ctx, g):
            x, wq = ctx.saved_tensors
            gq = q(g.reshape(-1, g.shape[-1])).reshape(g.shape)  # one scale per token
            return gq @ wq, (g.reshape(-1, g.shape[-1]).T @ x.reshape(-1, x.shape[-1]))

    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in params.items()}
    B, T = tok.shape
    d, H, hd, Hkv = w.d_model, w.n_head, w.head_dim, w.n_kv_head or w.n_head
    pos = torch.arange(T)
    mask = pos[None, :] <= pos[:, None]
    if w.window:
        mask &= (pos[:, None] - pos[None, :]) < w.window
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
        qkv = Fp8Linear.apply(norm(x), t[f"layers.{l}.wqkv"])
        qq, kk, vv = qkv.split([d, Hkv * hd, Hkv * hd], dim=-1)
        qq = norm(rot(qq.view(B, T, H, hd)))
        kk = norm(rot(kk.view(B, T, Hkv, hd)))
        vv = vv.view(B, T, Hkv, hd)
        o = F.scaled_dot_product_attention(qq.transpose(1, 2), kk.transpose(1, 2), vv.transpose(1, 2),
                                           attn_mask=mask, enable_gqa=True)
        x = x + Fp8Linear.apply(o.transpose(1, 2).reshape(B, T, d), t[f"layers.{l}.wo"])
        u = Fp8Linear.apply(norm(x), t[f"layers.{l}.wup"])
        x = x + Fp8Linear.apply(torch.relu(u).square(), t[f"layers.{l}.wdown"])
    z = F.linear(norm(x), t["lm_head"])
    loss = F.cross_entropy(z.view(B * T, -1), torch.tensor(tgt, dtype=torch.long).view(-1))
    loss.backward()
    return float(loss), {k: v.grad.numpy() for k, v in t.items()}


@pytest.mark.parametrize("kw", [dict(n_layer=2, seq_len=48, batch=2, vocab=512),
                                dict(n_layer=1, seq_len=33, batch=3, vocab=300, d_ff=320),
                                dict(n_layer=2, seq_len=40, batch=2, vocab=256, n_kv_head=2, window=9)])
def test_fp8_step_matches_torch_casts_and_straight_through(kw):
    w = synth.workload("story", fp8=True, **kw)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    res = oracle.step(oracle.from_workload(w), params, tok, tgt)
    tl, tg = _torch_fp8_step(w, params, tok, tgt)
    assert math.isclose(res.loss, tl, rel_tol=1e-12)
    for k in params:
        err = np.max(np.abs(res.grads[k] - tg[k])) / np.max(np.abs(tg[k]))
        assert err <= 1e-10, (k, err)


def test_fp8_model_close_to_bf16_model():
    w = synth.workload("story", n_layer=2, seq_len=64, batch=2)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    a = oracle.step(oracle.from_workload(w), params, tok, tgt)
    b = oracle.step(oracle.from_workload(w.replace(fp8=True)), params, tok, tgt)
    assert a.loss != b.loss and abs(a.loss - b.loss) / a.loss < 1e-2
    for k in params:
        g, r = b.grads[k].ravel(), a.grads[k].ravel()
        assert g @ r / (np.linalg.norm(g) * np.linalg.norm(r)) > 0.99, k
