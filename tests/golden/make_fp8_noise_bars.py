"""Size the full-size FP8 per-position loss bar from the oracle alone.

The e4m3 forward projections decide a code (and a per-row power-of-two scale)
from a bf16 activation.  The GPU forms that activation through its own bf16
pipeline, the oracle by rounding an fp64 value to bf16, so the two quantizer
inputs can differ in the last bf16 bit and then take different codes.  This
script measures how far that alone moves the oracle's per-position losses:
it runs the oracle's forward of the depth-24 FP8 workload over all 16
sequences (32,768 positions) with every quantizer input multiplied by
(1 + 1e-3 * N(0, 1)) -- about the relative deviation a bf16 pipeline carries
against fp64 -- and compares the per-position losses with the unperturbed
oracle's, read from ``oracle_samples_d24_fp8.npz`` (written by
``make_oracle_samples.py``).  The relative difference is the parity test's:
|a - b| / max(|b|, 1).

Calls only ``oracle`` and ``synth``; the perturbation wraps the oracle's
row quantizer from the outside and changes none of its arithmetic.  Output:
``fp8_noise_d24.json`` (the distribution and the bar derived from it).

Usage: python tests/golden/make_fp8_noise_bars.py
"""
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import oracle.gpt_oracle as G  # noqa: E402
import synth  # noqa: E402

NOISE = 1e-3
SEED = 7
# the bar: the emulated worst case with a factor of 1.5 for what one noise
# draw over 32,768 positions cannot show of the tail
BAR_FACTOR = 1.5


def main():
    w = synth.workload("d24", fp8=True)
    cfg = oracle.from_workload(w)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    clean = np.load(os.path.join(HERE, "oracle_samples_d24_fp8.npz"))["token_loss"]

    rng = np.random.Generator(np.random.PCG64(SEED))
    quantize = G.fp8_rows

    def noisy_rows(x):
        return quantize(x * (1.0 + NOISE * rng.standard_normal(x.shape)))

    G.fp8_rows = noisy_rows
    try:
        t0 = time.time()
        res = oracle.step(cfg, params, tok, tgt, backward=False)
        dt = time.time() - t0
    finally:
        G.fp8_rows = quantize

    rel = np.abs(res.token_loss - clean) / np.maximum(np.abs(clean), 1.0)
    q = [50, 90, 99, 99.9, 99.99, 100]
    out = {
        "workload": "d24 with e4m3 forward block projections, 16 x 2048 positions",
        "noise": f"quantizer input x (1 + {NOISE} N(0,1)), PCG64({SEED})",
        "positions": int(rel.size),
        "loss_clean": float(np.sum(clean) / clean.size),
        "loss_noisy": float(res.loss),
        "loss_rel_change": float(abs(res.loss - np.sum(clean) / clean.size) / (np.sum(clean) / clean.size)),
        "token_rel_quantiles": {str(p): float(np.percentile(rel, p)) for p in q},
        "count_above": {str(t): int(np.sum(rel > t)) for t in (1e-2, 2e-2, 4e-2, 6e-2)},
        "bar_factor": BAR_FACTOR,
        "token_bar": float(BAR_FACTOR * rel.max()),
        "oracle_seconds": dt,
    }
    path = os.path.join(HERE, "fp8_noise_d24.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
