"""Host-side logic of bench.py (CPU): the FLOP model, the roofline object, the
workload builder and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_flops_per_token_plain_model_closed_form():
    w = synth.workload("d24")
    L, d, V, T = w.n_layer, w.d_model, w.vocab, w.seq_len
    assert bench.flops_per_token(w) == 6.0 * (12 * L * d * d + V * d) + 6.0 * L * T * d


def _brute_visible_keys(T, W):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    vis = (j <= i) & ((i - j) < W if W else True)
    return vis.sum() / T


@pytest.mark.parametrize("T,W", [(64, 16), (100, 1), (128, 127), (50, 50)])
def test_flops_per_token_window_counts_visible_pairs(T, W):
    w = synth.workload("story", seq_len=T, window=W)
    L, d = w.n_layer, w.d_model
    base = synth.workload("story", seq_len=T)
    # only the attention term changes: 12 L d * (visible keys per query)
    delta = bench.flops_per_token(base) - bench.flops_per_token(w)
    want = 12.0 * L * d * (T / 2 - _brute_visible_keys(T, W)) if W < T else 0.0
    assert delta == pytest.approx(want, rel=1e-12, abs=1e-6)


def test_flops_per_token_gqa_shrinks_the_qkv_projection():
    w = synth.workload("d24")
    g = w.replace(n_kv_head=4)
    L, d, hd = w.n_layer, w.d_model, w.head_dim
    # q/k/v weights (d + 2 n_kv hd) d instead of 3 d d, times 6 (fwd + bwd)
    assert bench.flops_per_token(w) - bench.flops_per_token(g) == pytest.approx(
        6.0 * L * (2 * d - 2 * 4 * hd) * d)


def test_roofline_uses_the_site_and_the_dtype_peak():
    w = synth.workload("d24")
    sites = {"up_fwd": {"ms_per_launch": 0.5, "flops_per_launch": 6.0e11}}
    peaks = {"source": "measured"}
    r = bench.roofline(sites, w, 1300.0, 1400.0, peaks)
    assert r["achieved"] == pytest.approx(1200.0) and r["frac"] == pytest.approx(1200.0 / 1400.0, rel=1e-3)
    assert r["unit"] == "TFLOP/s" and r["bound"] == "tensor" and "traffic" in r
    f = bench.roofline(sites, w.replace(fp8=True), 1300.0, 1400.0, peaks)
    assert f["peak"] == 2800.0 and f["frac"] == pytest.approx(1200.0 / 2800.0, rel=1e-3)
    # DRAM traffic from the ncu captures of the d24 launches, below the
    # algorithmic bytes (no re-reads); other shapes have none
    assert r["traffic"] == 482_792_960 and r["traffic"] <= r["algorithmic_bytes_per_launch"]
    assert f["traffic"] == 412_028_416 and f["traffic"] <= f["algorithmic_bytes_per_launch"]
    assert bench.roofline(sites, synth.workload("d12"), 1300.0, 1400.0, peaks)["traffic"] is None


def test_workload_builder_applies_overrides():
    import argparse
    ns = argparse.Namespace(workload="d24", batch=4, layers=2, kv_heads=4, window=512, fp8=True)
    w = bench.bench_workload(ns)
    assert (w.batch, w.n_layer, w.n_kv_head, w.window, w.fp8) == (4, 2, 4, 512, True)
    desc = bench.workload_desc(w)
    assert "4 key/value heads" in desc and "window 512" in desc and "e4m3" in desc


def test_reference_arm_json_line():
    # the reference arm times the fp64 oracle on the host: one short sample of
    # the tiny workload, one JSON line with the contract's keys
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
