"""Write fp64 oracle outputs for a full-size workload to oracle_samples_<name>.npz.

Calls only ``oracle`` and ``synth``.  Stored: the loss, every per-position loss
[B, T], and for every parameter tensor the gradient at seeded coordinates
(PCG64(seed + 2000)) together with the tensor's Frobenius norm and max |g|.
For ``wte`` half the coordinates are on rows that some token hits and half on
rows that none hits (whose gradient must be exactly zero).

Usage: python tests/golden/make_oracle_samples.py d12 [d24 d24_kv4_w1024 ...]
(a name is a workload, or one of VARIANTS: a workload with model overrides).
"""
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import synth  # noqa: E402

SAMPLES_PER_TENSOR = 1024

# variants at full size: grouped-query attention with 4 key/value heads and a
# 1024-position sliding window on the d24 model; the d24 model with e4m3
# forward block projections
VARIANTS = {
    "d24_kv4_w1024": ("d24", dict(n_kv_head=4, window=1024)),
    "d24_fp8": ("d24", dict(fp8=True)),
    # the block variants at full size: value embeddings on every other layer,
    # residual scaling, smear and backout
    "d24_variants": ("d24", dict(ve_every=2, resid_lambdas=True, smear=True, backout=True)),
}


def workload_of(name):
    if name in VARIANTS:
        base, kw = VARIANTS[name]
        return synth.workload(base, **kw)
    return synth.workload(name)


def sample_coords(w, name, shape, tokens, rng):
    rows, cols = shape
    if name == "wte":
        hit = np.unique(tokens)
        miss = np.setdiff1d(np.arange(rows), hit)
        nh = SAMPLES_PER_TENSOR // 2
        r = np.concatenate([rng.choice(hit, nh), rng.choice(miss, SAMPLES_PER_TENSOR - nh)
                            if miss.size else rng.choice(hit, SAMPLES_PER_TENSOR - nh)])
    else:
        r = rng.integers(0, rows, SAMPLES_PER_TENSOR)
    c = rng.integers(0, cols, SAMPLES_PER_TENSOR)
    return r.astype(np.int64), c.astype(np.int64)


def main(name):
    w = workload_of(name)
    cfg = oracle.from_workload(w)
    tok, tgt = synth.make_tokens(w)
    params = synth.make_params(w)
    t0 = time.time()
    res = oracle.step(cfg, params, tok, tgt)
    dt = time.time() - t0
    rng = np.random.Generator(np.random.PCG64(w.seed + 2000))
    out = {"loss": np.float64(res.loss), "token_loss": res.token_loss,
           "oracle_seconds": np.float64(dt)}
    for pname, shape in synth.param_shapes(w):
        g = res.grads[pname]
        r, c = sample_coords(w, pname, shape, tok, rng)
        out[f"{pname}/rows"] = r
        out[f"{pname}/cols"] = c
        out[f"{pname}/values"] = g[r, c]
        out[f"{pname}/fro"] = np.float64(np.linalg.norm(g))
        out[f"{pname}/absmax"] = np.float64(np.max(np.abs(g)))
    path = os.path.join(HERE, f"oracle_samples_{name}.npz")
    np.savez_compressed(path, **out)
    print(f"{name}: loss {res.loss:.6f}, oracle {dt:.0f} s -> {path}")


if __name__ == "__main__":
    for n in sys.argv[1:] or ["d12"]:
        main(n)
