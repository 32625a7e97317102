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
* Coefficients are the caller's; the library's default schedule is the two
  printed triples followed by the second one repeated (the page's list breaks
  off after two entries).
* The NorMuon variance rescale is not built: its printed fragment uses names
  it never defines (red_dim, v_norm_new, step_size).
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


def muon(theta, g, mom, lr: float, mu: float, nesterov: bool,
         coeffs: Sequence[Tuple[float, float, float]]):
    """One Muon step on a [rows, cols] matrix.  Returns (theta, mom, x_final)."""
    theta = np.asarray(theta, np.float64)
    g = np.asarray(g, np.float64)
    mom = mu * np.asarray(mom, np.float64) + g
    u = g + mu * mom if nesterov else mom
    x = newton_schulz(u, coeffs)
    rows, cols = theta.shape
    scale = math.sqrt(max(1.0, rows / cols))
    return theta - lr * scale * x, mom, x


def is_muon(name: str) -> bool:
    """Block matrices go to Muon; the embedding and lm_head to AdamW."""
    return name.startswith("layers.")


def optimizer_step(master: Dict[str, np.ndarray], grads: Dict[str, np.ndarray],
                   m: Dict[str, np.ndarray], v: Dict[str, np.ndarray], hp: dict):
    """One optimizer step over every tensor.  ``hp`` keys: adam_lr, beta1,
    beta2, eps, weight_decay, muon_lr, momentum, nesterov, coeffs, step.
    For Muon tensors ``m`` holds the momentum and ``v`` is unused.
    Returns new (master, m, v) dicts (float64)."""
    out_w, out_m, out_v = {}, {}, {}
    for name, w in master.items():
        if is_muon(name):
            w2, mom, _ = muon(w, grads[name], m[name], hp["muon_lr"], hp["momentum"],
                              bool(hp["nesterov"]), hp["coeffs"])
            out_w[name], out_m[name], out_v[name] = w2, mom, np.asarray(v[name], np.float64)
        else:
            w2, m2, v2 = adamw(w, grads[name], m[name], v[name], hp["step"], hp["adam_lr"],
                               hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])
            out_w[name], out_m[name], out_v[name] = w2, m2, v2
    return out_w, out_m, out_v
