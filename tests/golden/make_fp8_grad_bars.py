"""Size the full-size FP8 gradient bars from the oracle alone.

The full-size FP8 parity check compares the GPU's d24 gradients (e4m3 forward
projections and data gradients) with stored oracle samples.  Where the GPU's
and the oracle's bf16 quantizer inputs differ in the last bit they can take
different e4m3 codes, and the gradients carry those code steps.  This script
measures how far that alone moves the oracle's d24 gradients: two sequences
of the d24 FP8 workload (with the full batch's 1/(B*T) factor), every input of
the oracle's row quantizer -- the forward's activations and the data
gradients' output gradients -- multiplied by (1 + 1e-3 * N(0, 1)), against
the same sequences unperturbed; per tensor the cosine and max-rel of the
parity test.  An embedding row sums only the few positions holding its token,
so its noise does not average out over more sequences: two sequences already
show the worst case of the full batch there.  The bars are the worst tensor
times BAR_FACTOR.

Calls only ``oracle`` and ``synth``; the perturbation wraps the oracle's row
quantizer from the outside and changes none of its arithmetic.  Output:
``fp8_noise_d24_grads.json``.

Usage: python tests/golden/make_fp8_grad_bars.py
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
ROWS = (0, 1)
BAR_FACTOR = 2.0


def metrics(g, r):
    g, r = g.ravel(), r.ravel()
    cos = float(g @ r / (np.linalg.norm(g) * np.linalg.norm(r) + 1e-300))
    return cos, float(np.max(np.abs(g - r)) / (np.max(np.abs(r)) + 1e-300))


def main():
    w = synth.workload("d24", fp8=True)
    cfg = oracle.from_workload(w)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    t0 = time.time()
    clean = oracle.step(cfg, params, tok, tgt, rows=ROWS)
    plain = G.fp8_rows
    rng = np.random.Generator(np.random.PCG64(SEED))
    G.fp8_rows = lambda x: plain(x * (1.0 + NOISE * rng.standard_normal(x.shape)))
    try:
        noisy = oracle.step(cfg, params, tok, tgt, rows=ROWS)
    finally:
        G.fp8_rows = plain
    per = {k: metrics(noisy.grads[k], clean.grads[k]) for k in clean.grads}
    worst_cos = min(per.items(), key=lambda kv: kv[1][0])
    worst_mr = max(per.items(), key=lambda kv: kv[1][1])
    out = {
        "workload": "d24 with e4m3 block projections (forward and data gradients), sequences 0 and 1",
        "noise": f"row-quantizer input x (1 + {NOISE} N(0,1)), PCG64({SEED})",
        "worst_cos": {"tensor": worst_cos[0], "cos": worst_cos[1][0]},
        "worst_maxrel": {"tensor": worst_mr[0], "maxrel": worst_mr[1][1]},
        "per_tensor": {k: {"cos": v[0], "maxrel": v[1]} for k, v in sorted(per.items())},
        "bar_factor": BAR_FACTOR,
        "bars": {"cos": 1.0 - BAR_FACTOR * (1.0 - worst_cos[1][0]), "maxrel": BAR_FACTOR * worst_mr[1][1]},
        "oracle_seconds": time.time() - t0,
    }
    with open(os.path.join(HERE, "fp8_noise_d24_grads.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps({k: out[k] for k in ("worst_cos", "worst_maxrel", "bars", "oracle_seconds")}, indent=1))


if __name__ == "__main__":
    main()
