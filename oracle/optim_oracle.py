"""fp64 CPU oracle for the optimizer step that follows the backward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check in
``__graft_entry__`` and ``bench.py``'s CPU-baseline / reference arm may import
this module; the CUDA library never calls it and shares no code with it.

What the pages fix
------------------
"ChatGPT'nizi 50 Dolara Nasil Egitirsiniz?" (dev.to), section "2. Muon
Optimize Edici (nanochat/optim.py)":

* the embeddings and lm_head are updated with AdamW, the 2-D block matrices
  with Muon (momentum orthogonalised by a Newton-Schulz iteration);
* one orthogonalisation iteration with coefficients (a, b, c) is
  A = X^T X,  B = b A + c A A,  X <- a X + X B;
* the "Polar Express" schedule has five (a, b, c) triples, of which the page
  prints the first two, (8.156, -22.483, 15.879) and (4.043, -2.809, 0.500).

AdamW itself is the published algorithm (Adam's moment estimates with bias
correction and decoupled weight decay, Loshchilov and Hutter).

Readings where the pages are silent or the text breaks off
----------------------------------------------------------
* Master weights: the page's ``F.linear(x, W.to(x.dtype))`` (section "3.
  Hassasiyet Yonetimi") casts a higher-precision W to bf16 per call, so the
  optimizer updates an fp32/fp64 master copy; the bf16 parameters are that
  copy rounded after each step.
* AdamW: m <- b1 m + (1-b1) g;  v <- b2 v + (1-b2) g^2;
  theta <- theta (1 - lr wd) - lr (m / (1-b1^t)) / (sqrt(v / (1-b2^t)) + eps).
* Muon: M <- mu M + G;  U = G + mu M with Nesterov momentum, else U = M;
  X0 = U / (||U||_F + 1e-7);  the Newton-Schulz iterations as printed, with
  the Gram matrix over the smaller dimension (for a wide X the same map is
  applied to X^T: A = X X^T, X <- a X + B X);  theta <- theta - lr s X_final
  with s = sqrt(max(1, rows / cols)); no weight decay on these matrices.
* Coefficients are the caller's.  The library's default schedule is the two
  printed triples only (ns_steps = 2); ``default_coeffs(n)`` here pads a
  longer test schedule with the last printed triple (the page's list breaks
  off after two entries).
* NorMuon (same section, "NorMuon Varyans Azaltma"): the page prints the
  rescale of the orthogonalised update g as four lines that use three names
  it never defines (red_dim, step_size, v_norm_new).  Reading, after the
  published NorMuon method (Li et al., 2025: one second-moment estimate per
  output neuron of the orthogonalised update, the update normalised by it):
    - red_dim is the column dimension: v_mean[r] = mean_c g[r, c]^2, one per
      row (output neuron) of the [out, in] matrix;
    - v_norm = sqrt(sum_r v_mean[r]), as printed;
    - a per-row state buf (fp32, zero at init) follows the EMA
      buf <- beta2 buf + (1 - beta2) v_mean, beta2 = 0.95 by default (the
      published method's value); step_size[r] = 1 / sqrt(max(buf[r], 1e-10));
    - v_norm_new is the same statistic of the rescaled update g * step_size:
      sqrt(sum_r v_mean[r] step_size[r]^2);
    - final_scale[r] = step_size[r] v_norm / max(v_norm_new, 1e-10) and
      g <- g * final_scale, as printed: each row keeps its direction and the
      update keeps its Frobenius norm, only its spread over the rows changes.
  The Muon update then uses the rescaled g.
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, Sequence, Tuple

import numpy as np

__all__ = [
    "PRINTED_COEFFS",
    "default_coeffs",
    "adamw",
    "ns_iteration",
    "newton_schulz",
    "normuon",
    "muon",
    "optimizer_step",
    "is_muon",
]

# the two triples the page prints, in its order
PRINTED_COEFFS: Tuple[Tuple[float, float, float], ...] = (
    (8.156, -22.483, 15.879),
    (4.043, -2.809, 0.500),
)


def default_coeffs(ns_steps: int = 5):
    """The printed triples, then the last printed one repeated."""
    out = list(PRINTED_COEFFS[:ns_steps])
    while len(out) < ns_steps:
        out.append(PRINTED_COEFFS[-1])
    return out


def adamw(theta, g, m, v, t: int, lr: float, b1: float, b2: float, eps: float, wd: float):
    """One AdamW step (bias-corrected moments, decoupled weight decay).
    Returns (theta, m, v), all float64."""
    theta = np.asarray(theta, np.float64)
    g = np.asarray(g, np.float64)
    m = b1 * np.asarray(m, np.float64) + (1.0 - b1) * g
    v = b2 * np.asarray(v, np.float64) + (1.0 - b2) * g * g
    m_hat = m / (1.0 - b1 ** t)
    v_hat = v / (1.0 - b2 ** t)
    theta = theta * (1.0 - lr * wd) - lr * m_hat / (np.sqrt(v_hat) + eps)
    return theta, m, v


def ns_iteration(x: np.ndarray, a: float, b: float, c: float) -> np.ndarray:
    """One orthogonalisation iteration as the page prints it, with the Gram
    matrix taken over the smaller dimension."""
    x = np.asarray(x, np.float64)
    if x.shape[0] >= x.shape[1]:
        A = x.T @ x
        B = b * A + c * (A @ A)
        return a * x + x @ B
    A = x @ x.T
    B = b * A + c * (A @ A)
    return a * x + B @ x


def newton_schulz(u: np.ndarray, coeffs: Sequence[Tuple[float, float, float]]) -> np.ndarray:
    """Frobenius-normalise, then iterate."""
    u = np.asarray(u, np.float64)
    x = u / (np.linalg.norm(u) + 1e-7)
    for a, b, c in coeffs:
        x = ns_iteration(x, a, b, c)
    return x


def normuon(x: np.ndarray, buf: np.ndarray, beta2: float):
    """The NorMuon rescale of an orthogonalised update x [rows, cols] with the
    per-row second-moment state buf [rows] (reading in the module docstring).
    Returns (x rescaled, new buf)."""
    x = np.asarray(x, np.float64)
    v_mean = np.mean(x * x, axis=1)                       # red_dim: the columns
    v_norm = math.sqrt(float(np.sum(v_mean)))
    buf = beta2 * np.asarray(buf, np.float64) + (1.0 - beta2) * v_mean
    step_size = 1.0 / np.sqrt(np.maximum(buf, 1e-10))
    v_norm_new = math.sqrt(float(np.sum(v_mean * step_size * step_size)))
    final_scale = step_size * (v_norm / max(v_norm_new, 1e-10))
    return x * final_scale[:, None], buf


def muon(theta, g, mom, lr: float, mu: float, nesterov: bool,
         coeffs: Sequence[Tuple[float, float, float]], normuon_buf=None, normuon_beta2: float = 0.95):
    """One Muon step on a [rows, cols] matrix.  With ``normuon_buf`` (the
    per-row state) the orthogonalised update is NorMuon-rescaled first.
    Returns (theta, mom, x_final, new normuon_buf or None)."""
    theta = np.asarray(theta, np.float64)
    g = np.asarray(g, np.float64)
    mom = mu * np.asarray(mom, np.float64) + g
    u = g + mu * mom if nesterov else mom
    x = newton_schulz(u, coeffs)
    buf = None
    if normuon_buf is not None:
        x, buf = normuon(x, normuon_buf, normuon_beta2)
    rows, cols = theta.shape
    scale = math.sqrt(max(1.0, rows / cols))
    return theta - lr * scale * x, mom, x, buf


def is_muon(name: str) -> bool:
    """Block matrices go to Muon; the embedding and lm_head to AdamW."""
    return name.startswith("layers.")


def optimizer_step(master: Dict[str, np.ndarray], grads: Dict[str, np.ndarray],
                   m: Dict[str, np.ndarray], v: Dict[str, np.ndarray], hp: dict):
    """One optimizer step over every tensor.  ``hp`` keys: adam_lr, beta1,
    beta2, eps, weight_decay, muon_lr, momentum, nesterov, coeffs, step, and
    optionally normuon (bool) and normuon_beta2.  For Muon tensors ``m``
    holds the momentum and ``v`` the NorMuon state in its first ``rows``
    entries (flattened; the rest unused, as the library's state buffer).
    Returns new (master, m, v) dicts (float64)."""
    out_w, out_m, out_v = {}, {}, {}
    for name, w in master.items():
        if is_muon(name):
            vv = np.array(v[name], np.float64)
            rows = w.shape[0]
            buf = vv.ravel()[:rows] if hp.get("normuon") else None
            w2, mom, _, buf = muon(w, grads[name], m[name], hp["muon_lr"], hp["momentum"],
                                   bool(hp["nesterov"]), hp["coeffs"], buf,
                                   hp.get("normuon_beta2", 0.95))
            if buf is not None:
                flat = vv.ravel()
                flat[:rows] = buf
                vv = flat.reshape(vv.shape)
            out_w[name], out_m[name], out_v[name] = w2, mom, vv
        else:
            w2, m2, v2 = adamw(w, grads[name], m[name], v[name], hp["step"], hp["adam_lr"],
                               hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])
            out_w[name], out_m[name], out_v[name] = w2, m2, v2
    return out_w, out_m, out_v
