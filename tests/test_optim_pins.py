"""Pins for the optimizer oracle (CPU): each check comes from mathematics or an
independent library routine, not from re-typing the oracle's formulas.

Sources: "ChatGPT'nizi 50 Dolara Nasil Egitirsiniz?", section "2. Muon
Optimize Edici (nanochat/optim.py)" (the Newton-Schulz iteration and its first
two Polar Express coefficient triples); AdamW as published (bias-corrected
Adam moments, decoupled weight decay).
"""
import math

import numpy as np
import pytest

from oracle import optim_oracle as O


def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("shape", [(7, 4), (4, 7), (5, 5)])
def test_ns_iteration_acts_on_singular_values(shape):
    # On X = U diag(s) V^T one iteration maps each singular value s to the odd
    # quintic p(s) = a s + b s^3 + c s^5 and keeps U, V (page's iteration with
    # its first printed triple).
    a, b, c = O.PRINTED_COEFFS[0]
    rng = _rng(1)
    r, k = shape
    n = min(r, k)
    U, _ = np.linalg.qr(rng.standard_normal((r, n)))
    V, _ = np.linalg.qr(rng.standard_normal((k, n)))
    s = rng.uniform(0.05, 1.0, n)
    x = U @ np.diag(s) @ V.T
    want = U @ np.diag(a * s + b * s ** 3 + c * s ** 5) @ V.T
    np.testing.assert_allclose(O.ns_iteration(x, a, b, c), want, atol=1e-12)


def test_printed_triples_expand_small_singular_values():
    # both printed polynomials have slope a > 1 at 0, so they push small
    # singular values up, as an orthogonalising schedule must: p(s) > s
    for a, b, c in O.PRINTED_COEFFS:
        for s in (1e-3, 1e-2, 0.05):
            assert a * s + b * s ** 3 + c * s ** 5 > s


def test_classic_newton_schulz_converges_to_polar_factor():
    # with (1.5, -0.5, 0) the iteration is the cubic Newton-Schulz map, whose
    # fixed point for a full-rank X with singular values in (0, sqrt(3)) is the
    # orthogonal polar factor U V^T (checked against numpy's SVD)
    rng = _rng(2)
    for shape in ((24, 16), (16, 24)):
        x = rng.standard_normal(shape)
        U, s, Vt = np.linalg.svd(x, full_matrices=False)
        polar = U @ Vt
        got = O.newton_schulz(x, [(1.5, -0.5, 0.0)] * 60)
        np.testing.assert_allclose(got, polar, atol=1e-9)


def test_newton_schulz_transpose_equivariant():
    rng = _rng(3)
    x = rng.standard_normal((12, 20))
    coeffs = O.default_coeffs(5)
    np.testing.assert_allclose(O.newton_schulz(x.T, coeffs), O.newton_schulz(x, coeffs).T, atol=1e-10)


def test_newton_schulz_orthogonal_invariance():
    # a matrix function of the singular values: ns(Q X R) = Q ns(X) R
    rng = _rng(4)
    x = rng.standard_normal((10, 6))
    Q, _ = np.linalg.qr(rng.standard_normal((10, 10)))
    R, _ = np.linalg.qr(rng.standard_normal((6, 6)))
    coeffs = O.default_coeffs(5)
    np.testing.assert_allclose(O.newton_schulz(Q @ x @ R, coeffs), Q @ O.newton_schulz(x, coeffs) @ R,
                               atol=1e-10)


def test_default_schedule():
    cs = O.default_coeffs(5)
    assert cs[0] == (8.156, -22.483, 15.879) and cs[1] == (4.043, -2.809, 0.500)
    assert cs[2:] == [cs[1]] * 3
    assert O.default_coeffs(1) == [cs[0]]


def test_adamw_first_step_closed_form():
    # t = 1: m_hat = g and v_hat = g^2, so the step is lr * g / (|g| + eps)
    rng = _rng(5)
    theta = rng.standard_normal(50)
    g = rng.standard_normal(50)
    lr, wd, eps = 3e-3, 0.1, 1e-8
    got, m, v = O.adamw(theta, g, np.zeros(50), np.zeros(50), 1, lr, 0.8, 0.95, eps, wd)
    want = theta * (1 - lr * wd) - lr * g / (np.abs(g) + eps)
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(m, 0.2 * g, rtol=1e-14)
    np.testing.assert_allclose(v, 0.05 * g * g, rtol=1e-14)  # 1 - 0.95 is not exactly 0.05 in fp64


def test_adamw_two_steps_by_hand():
    # scalar worked by hand: g1 = 2, g2 = -1, b1 = 0.5, b2 = 0.75, lr = 0.1,
    # eps = 0, wd = 0, theta0 = 1.
    # t=1: m = 1, v = 1, m_hat = 2, v_hat = 4 -> theta = 1 - 0.1 * 2/2 = 0.9
    # t=2: m = 0.5 - 0.5 = 0, so theta stays 0.9; v = 0.75 + 0.25 = 1
    th, m, v = O.adamw(1.0, 2.0, 0.0, 0.0, 1, 0.1, 0.5, 0.75, 0.0, 0.0)
    assert abs(th - 0.9) < 1e-15 and abs(m - 1.0) < 1e-15 and abs(v - 1.0) < 1e-15
    th, m, v = O.adamw(th, -1.0, m, v, 2, 0.1, 0.5, 0.75, 0.0, 0.0)
    assert abs(th - 0.9) < 1e-15 and abs(m) < 1e-15 and abs(v - 1.0) < 1e-15


def test_momentum_geometric_sum():
    # constant gradient G for k steps from zero: M_k = G (1 - mu^k) / (1 - mu)
    G = np.array([[1.0, -2.0], [0.5, 3.0]])
    mom = np.zeros_like(G)
    w = np.zeros_like(G)
    mu = 0.9
    for k in range(1, 6):
        w, mom, _, _ = O.muon(w, G, mom, 0.0, mu, False, O.default_coeffs(5))
        np.testing.assert_allclose(mom, G * (1 - mu ** k) / (1 - mu), rtol=1e-14)


def test_muon_step_on_orthogonal_gradient():
    # G with orthonormal columns: the normalised start has all singular values
    # 1/sqrt(cols); with the cubic map iterated to convergence the update is
    # -lr * sqrt(rows/cols) * G exactly (its polar factor is itself)
    rng = _rng(6)
    Qm, _ = np.linalg.qr(rng.standard_normal((9, 4)))
    w0 = rng.standard_normal((9, 4))
    w1, mom, x, _ = O.muon(w0, Qm, np.zeros((9, 4)), 0.01, 0.95, False, [(1.5, -0.5, 0.0)] * 40)
    np.testing.assert_allclose(x, Qm, atol=1e-10)
    np.testing.assert_allclose(w1, w0 - 0.01 * math.sqrt(9 / 4) * Qm, atol=1e-10)


def test_nesterov_direction():
    # one step from zero momentum: M = G and U = G + mu G, so the orthogonalised
    # direction is that of G either way (normalisation removes the scale; a
    # large gradient makes the 1e-7 in the normalisation negligible)
    rng = _rng(7)
    G = 1e4 * rng.standard_normal((6, 6))
    _, _, x1, _ = O.muon(np.zeros((6, 6)), G, np.zeros((6, 6)), 0.1, 0.9, True, O.default_coeffs(5))
    _, _, x0, _ = O.muon(np.zeros((6, 6)), G, np.zeros((6, 6)), 0.1, 0.9, False, O.default_coeffs(5))
    np.testing.assert_allclose(x1, x0, atol=1e-12)


def test_nesterov_two_steps_closed_form():
    # M1 = G1, M2 = mu G1 + G2, U2 = G2 + mu M2 = (1 + mu) G2 + mu^2 G1
    rng = _rng(9)
    G1, G2 = rng.standard_normal((5, 3)), rng.standard_normal((5, 3))
    mu, coeffs = 0.9, O.default_coeffs(5)
    w, mom, _, _ = O.muon(np.zeros((5, 3)), G1, np.zeros((5, 3)), 0.0, mu, True, coeffs)
    w, mom, x, _ = O.muon(w, G2, mom, 0.0, mu, True, coeffs)
    np.testing.assert_allclose(mom, mu * G1 + G2, rtol=1e-14)
    np.testing.assert_allclose(x, O.newton_schulz((1 + mu) * G2 + mu * mu * G1, coeffs), atol=1e-12)


def test_optimizer_step_routes_tensors():
    rng = _rng(8)
    master = {"wte": rng.standard_normal((5, 4)), "layers.0.wo": rng.standard_normal((4, 4)),
              "lm_head": rng.standard_normal((5, 4))}
    grads = {k: rng.standard_normal(v.shape) for k, v in master.items()}
    zeros = {k: np.zeros_like(v) for k, v in master.items()}
    hp = dict(adam_lr=1e-3, beta1=0.8, beta2=0.95, eps=1e-10, weight_decay=0.0, muon_lr=0.02,
              momentum=0.95, nesterov=1, coeffs=O.default_coeffs(5), step=1)
    w, m, v = O.optimizer_step(master, grads, zeros, zeros, hp)
    for k in ("wte", "lm_head"):
        want, _, _ = O.adamw(master[k], grads[k], zeros[k], zeros[k], 1, 1e-3, 0.8, 0.95, 1e-10, 0.0)
        np.testing.assert_allclose(w[k], want)
        assert np.all(v[k] > 0)
    want, _, _, _ = O.muon(master["layers.0.wo"], grads["layers.0.wo"], zeros["layers.0.wo"], 0.02, 0.95,
                        True, O.default_coeffs(5))
    np.testing.assert_allclose(w["layers.0.wo"], want)
    assert np.all(v["layers.0.wo"] == 0)


# ---- NorMuon rescale (reading of the fragment in "2. Muon Optimize Edici") --

def test_normuon_hand_worked_2x3():
    # x rows [1, 2, 2] and [0, 0, 1]: mean squares 3 and 1/3; beta2 = 0.5 from
    # a zero state gives buf = (1.5, 1/6), step sizes 1/sqrt(1.5) and sqrt(6);
    # v_norm = sqrt(10/3), v_norm_new = sqrt(3/1.5 + 6/3) = 2, so the rows are
    # scaled by sqrt(10/3)/2 * (1/sqrt(1.5), sqrt(6)) = (sqrt(5)/3, sqrt(5)):
    # both rows end with norm sqrt(5), and the total stays sqrt(10)
    x = np.array([[1.0, 2.0, 2.0], [0.0, 0.0, 1.0]])
    y, buf = O.normuon(x, np.zeros(2), 0.5)
    np.testing.assert_allclose(buf, [1.5, 1.0 / 6.0], rtol=1e-15)
    np.testing.assert_allclose(y, [[math.sqrt(5) / 3, 2 * math.sqrt(5) / 3, 2 * math.sqrt(5) / 3],
                                   [0.0, 0.0, math.sqrt(5)]], rtol=1e-14)


@pytest.mark.parametrize("shape", [(7, 5), (4, 11), (16, 16)])
def test_normuon_keeps_frobenius_norm_and_row_directions(shape):
    rng = _rng(21)
    x = rng.standard_normal(shape) * rng.uniform(0.1, 3.0, (shape[0], 1))
    buf0 = rng.uniform(0.0, 2.0, shape[0])
    y, _ = O.normuon(x, buf0, 0.9)
    assert abs(np.linalg.norm(y) / np.linalg.norm(x) - 1.0) < 1e-13
    # each row is a positive multiple of the input row
    ratio = np.sum(y * x, axis=1) / np.sum(x * x, axis=1)
    assert np.all(ratio > 0)
    np.testing.assert_allclose(y, ratio[:, None] * x, rtol=1e-12, atol=1e-15)


def test_normuon_equal_rows_from_zero_state_is_identity():
    # rows of equal mean square (an orthogonal matrix) from a zero state: every
    # step size is the same, so the norm-preserving rescale changes nothing
    rng = _rng(22)
    q, _ = np.linalg.qr(rng.standard_normal((6, 6)))
    y, buf = O.normuon(q, np.zeros(6), 0.95)
    np.testing.assert_allclose(y, q, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(buf, np.full(6, 0.05 / 6), rtol=1e-13)


def test_normuon_state_is_a_geometric_average():
    # the same update k times from a zero state: buf = (1 - beta2^k) mean_c x^2
    rng = _rng(23)
    x = rng.standard_normal((5, 4))
    buf = np.zeros(5)
    for k in range(1, 6):
        _, buf = O.normuon(x, buf, 0.8)
        np.testing.assert_allclose(buf, (1 - 0.8 ** k) * np.mean(x * x, axis=1), rtol=1e-14)


def test_normuon_zero_row_stays_zero():
    x = np.array([[0.0, 0.0, 0.0], [1.0, -1.0, 2.0]])
    y, buf = O.normuon(x, np.zeros(2), 0.95)
    assert np.all(np.isfinite(y)) and np.all(y[0] == 0)
    np.testing.assert_allclose(np.linalg.norm(y), np.linalg.norm(x), rtol=1e-14)


def test_optimizer_step_keeps_normuon_state_in_v():
    rng = _rng(24)
    master = {"layers.0.wup": rng.standard_normal((6, 4))}
    grads = {"layers.0.wup": rng.standard_normal((6, 4))}
    zeros = {"layers.0.wup": np.zeros((6, 4))}
    hp = dict(adam_lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, muon_lr=0.02,
              momentum=0.95, nesterov=1, coeffs=O.default_coeffs(2), step=1, normuon=True,
              normuon_beta2=0.9)
    w, m, v = O.optimizer_step(master, grads, zeros, zeros, hp)
    x = O.newton_schulz(grads["layers.0.wup"] * (1 + 0.95), O.default_coeffs(2))
    y, buf = O.normuon(x, np.zeros(6), 0.9)
    np.testing.assert_allclose(w["layers.0.wup"], master["layers.0.wup"] - 0.02 * math.sqrt(6 / 4) * y,
                               rtol=1e-13)
    np.testing.assert_allclose(v["layers.0.wup"].ravel()[:6], buf, rtol=1e-14)
    assert np.all(v["layers.0.wup"].ravel()[6:] == 0)
