#!/usr/bin/env python
"""Training-step throughput of the depth-24 GPT on B200 (tokens/s and MFU).

One step = gpt_forward_loss + gpt_backward (every gradient written, no
optimizer) on one synthetic batch of 16 x 2048 tokens (Zipf(1.1) ids, seeded
N(0, 0.02) bf16 weights).  Inputs are resident in HBM when the timed region
starts; the step touches tens of GB, far more than the 126 MB L2, so no L2
flush is needed between steps.  The headline region runs without the
per-launch trace; a second pass with the trace attached gives the per-kernel
breakdown.  Default runs also measure the depth-12 model (key "d12"), the
other depth the metric names.  MFU is against the nominal dense bf16 peak
(2.25 PFLOP/s), with the fraction of the measured sustained peak beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU runs (under torchrun) are replicas by default: every rank runs the
whole step on its own batch; ranks meet only at the timing barriers, and the
reported time is the maximum over ranks.  With --dp the ranks also sum their
gradients (data-parallel training, NCCL all-reduce per layer bucket,
overlapped with the backward).  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the only reference there is) on
the host cores, on a bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOAD = "d24"
SECOND_WORKLOAD = "d12"  # the metric names depth 12 and 24: d12 rides along in default runs
METRIC = "train tokens/sec (fwd+bwd) on 1 B200 for depth-12/24 GPT; MFU vs bf16 peak"


def flops_per_token(w) -> float:
    """Algorithmic FLOPs per token, fwd+bwd = 3x fwd: 6*(12 L d^2 + V d) + 6 L T d for the
    plain model (causal: T/2 keys per query on average).  With grouped-query attention the
    q/k/v projection has (d + 2 n_kv hd) d weights; with a sliding window W < T a query
    sees (W T - W (W-1)/2) / T keys on average."""
    L, d, V, T, F = w.n_layer, w.d_model, w.vocab, w.seq_len, w.d_ff
    qkv = d + 2 * (w.n_kv_head or w.n_head) * w.head_dim
    keys = T / 2
    if w.window and w.window < T:
        keys = (w.window * T - w.window * (w.window - 1) / 2) / T
    return 6.0 * (L * (qkv * d + d * d + 2 * F * d) + V * d) + 12.0 * L * keys * d


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16_tflops=p["bf16_tflops"],
                    bf16_tflops_sustained=p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def bench_workload(args):
    """The workload both arms run: the named one with the command line's
    model overrides (smaller profiling cases, the block and FP8 variants)."""
    w = synth.workload(args.workload)
    if args.batch:
        w = w.replace(batch=args.batch)
    if args.layers is not None:
        w = w.replace(n_layer=args.layers)
    if args.kv_heads:
        w = w.replace(n_kv_head=args.kv_heads)
    if args.window:
        w = w.replace(window=args.window)
    if args.fp8:
        w = w.replace(fp8=True)
    if getattr(args, "variants", False):
        w = w.replace(ve_every=2, resid_lambdas=True, smear=True, backout=True)
    return w


def workload_desc(w):
    extra = ""
    if w.n_kv_head and w.n_kv_head != w.n_head:
        extra += f", {w.n_kv_head} key/value heads"
    if w.window:
        extra += f", attention window {w.window}"
    if w.fp8:
        extra += ", e4m3 forward block projections"
    if w.ve_every or w.resid_lambdas or w.smear or w.backout:
        parts = ([f"value embeddings every {w.ve_every} layers"] if w.ve_every else []) + \
                (["residual scaling"] if w.resid_lambdas else []) + (["smear"] if w.smear else []) + \
                (["backout"] if w.backout else [])
        extra += ", " + ", ".join(parts)
    return (f"{w.name}: {w.n_layer} layers, d_model {w.d_model}, {w.n_head}x{w.head_dim} heads, "
            f"d_ff {w.d_ff}, vocab {w.vocab}, seq {w.seq_len}, batch {w.batch}{extra}")


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus = bus_id
        self.proc = None
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [r.split(", ") for r in self.tmp.read().strip().splitlines() if r.strip()]
        os.unlink(self.tmp.name)
        if self.bus:
            key = self.bus.lower()[-7:]
            rows = [r for r in rows if r and r[0].lower().endswith(key)] or rows
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_sample_setup(w, bits=None, target_s=10.0):
    """The oracle on the first n positions of one sequence of workload w, with n
    (a multiple of 32, at most seq_len) sized from a 32-position probe so that
    one sample takes about target_s seconds on this host."""
    import oracle
    if bits is None:
        bits = synth.make_params(w, as_bits=True)
    # bf16 workloads: the stored bit patterns; fp32 workloads: the fp32 values
    params = {k: synth.bf16_bits_to_f64(v) if w.dtype == "bf16" else np.asarray(v, dtype=np.float64)
              for k, v in bits.items()}
    tok, tgt = synth.make_tokens(w)

    def setup(n):
        ws = w.replace(seq_len=n, batch=1)
        return oracle, oracle.from_workload(ws), params, tok[:1, :n], tgt[:1, :n]

    probe = setup(min(32, w.seq_len))
    time_oracle(probe)                       # untimed: BLAS start-up, page-in
    per_tok = time_oracle(probe) / probe[3].shape[1]
    n = int(max(32, min(w.seq_len, round(target_s / per_tok / 32) * 32)))
    return setup(min(n, w.seq_len))


def time_oracle(setup, steps=1):
    oracle, cfg, params, tok, tgt = setup
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.step(cfg, params, tok, tgt)
    return time.perf_counter() - t0


def sample_tokens(setup):
    return int(setup[3].shape[1])


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def gemm_sites(records, w, steps):
    """Per-call-site GEMM time from the launch-ordered trace: the step launches
    forward [qkv, o, up, down] per layer then the lm_head statistics GEMM, and
    backward [logit grad, dhf, dWlm] then per layer (last first) [down dgrad,
    down wgrad, up dgrad, up wgrad, o dgrad, o wgrad, qkv dgrad, qkv wgrad]."""
    L = w.n_layer
    names = []
    for _ in range(L):
        names += ["qkv_fwd", "o_fwd", "up_fwd", "down_fwd"]
    names += ["lm_fwd_ce", "lm_grad_logits", "lm_dgrad", "lm_wgrad"]
    for _ in range(L):
        names += ["down_dgrad", "down_wgrad", "up_dgrad", "up_wgrad", "o_dgrad", "o_wgrad",
                  "qkv_dgrad", "qkv_wgrad"]
    gemms = [r for r in records if r[0] == "gemm"]
    if len(gemms) != len(names) * steps:
        return None
    acc = {}
    for i, (_, _, ms, fl, _) in enumerate(gemms):
        n = names[i % len(names)]
        a = acc.setdefault(n, [0.0, 0.0])
        a[0] += ms
        a[1] += fl
    return {n: {"ms_per_step": round(v[0] / steps, 3),
                "tflops": round(v[1] / (v[0] / 1e3) / 1e12, 1) if v[0] else None,
                "ms_per_launch": round(v[0] / (steps * names.count(n)), 4),
                "flops_per_launch": v[1] / (steps * names.count(n))}
            for n, v in acc.items()}


# DRAM bytes (read + write) of one launch of the dominant kernel's roofline
# site, from an ncu capture of the current kernel build, keyed by (workload,
# site, fp8); a site that has not been captured reports null.
TRAFFIC_BYTES = {
    ("d24", 32768, 6144, 1536, False): 121_198_336 + 361_594_624,  # ncu: 482.8 MB per launch
    ("d24", 32768, 6144, 1536, True): 60_164_608 + 351_863_808,    # e4m3 operands: 412.0 MB
}


def roofline(sites, w, gemm_tf, peak_tf, peaks):
    """Roofline of the dominant kernel, the tcgen05 CTA-pair GEMM: its
    up-projection forward launch (M = B*T, N = d_ff, K = d_model, ReLU^2
    epilogue), timed by the trace pass's CUDA events on the launching stream;
    the all-launch GEMM figure rides along."""
    site = (sites or {}).get("up_fwd")
    line = {"bound": "tensor", "kernel": "gemm_pair_kernel (tcgen05 cta_group::2 GEMM)",
            "site": f"up-projection forward: M={w.batch * w.seq_len} N={w.d_ff} K={w.d_model}",
            "peak": peak_tf, "unit": "TFLOP/s",
            "peak_source": f"{peaks['source']} bf16_tflops_sustained (kernel timed inside a long step)",
            "all_gemm_launches": {"achieved": round(gemm_tf, 1), "frac": round(gemm_tf / peak_tf, 4)}}
    site_peak = peak_tf
    if w.fp8:
        # the site runs on e4m3 operands: the measured bf16 peak times the
        # nominal e4m3 / bf16 dense ratio (4.5 / 2.25 PFLOP/s)
        site_peak = 2.0 * peak_tf
        line.update({"kernel": "gemm_pair_kernel (tcgen05 cta_group::2 GEMM, kind::f8f6f4 e4m3)",
                     "peak": site_peak,
                     "peak_source": f"{peaks['source']} bf16_tflops_sustained x 2 (nominal e4m3/bf16 ratio)",
                     "all_gemm_launches": {"achieved": round(gemm_tf, 1), "mixed": "e4m3 forward and data gradients, bf16 weight gradients"}})
    if site and site["ms_per_launch"] > 0:
        tf = site["flops_per_launch"] / (site["ms_per_launch"] / 1e3) / 1e12
        key = (w.name, w.batch * w.seq_len, w.d_ff, w.d_model, bool(w.fp8))
        line.update({"achieved": round(tf, 1), "frac": round(tf / site_peak, 4),
                     "algorithmic_flops_per_launch": site["flops_per_launch"],
                     "algorithmic_bytes_per_launch": (1 if w.fp8 else 2) * (w.batch * w.seq_len * w.d_model
                                                                           + w.d_ff * w.d_model)
                                                     + 2 * w.batch * w.seq_len * w.d_ff,
                     "traffic": TRAFFIC_BYTES.get(key)})
    else:
        line.update({"achieved": round(gemm_tf, 1), "frac": round(gemm_tf / site_peak, 4), "traffic": None})
    return line


def time_optimizer(B, st, stream, reps=3):
    """Device time of gpt_optim_step on the step's own gradients (library
    defaults: the two printed Newton-Schulz iterations), with the per-class
    trace: the Newton-Schulz GEMMs and the element-wise AdamW / Muon passes."""
    import torch
    opt = B.optim_defaults()
    st.init_optimizer()
    st.optimizer_step(opt)  # warm-up
    torch.cuda.synchronize()
    trace = B.Trace(capacity=8192)
    trace.attach()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(reps):
        opt.step = 2 + i
        st.optimizer_step(opt)
    e1.record(stream)
    torch.cuda.synchronize()
    B.Trace.detach()
    stats, _ = trace.summary()
    trace.close()
    code = st.status()
    if code != B.GPT_OK:
        raise SystemExit(f"device status after optimizer steps: {B.strerror(code)}")
    ms = e0.elapsed_time(e1) / reps
    g, o = stats["gemm"], stats["other"]
    line = {"ms_per_step": round(ms, 3), "ns_steps": int(opt.ns_steps),
            "state_bytes": int(st.opt_state.numel()),
            "newton_schulz_gemm": {"ms_per_step": round(g["ms"] / reps, 3),
                                   "launches_per_step": g["launches"] // reps,
                                   "tflops": round(g["flops"] / (g["ms"] / 1e3) / 1e12, 1) if g["ms"] else None},
            "elementwise": {"ms_per_step": round(o["ms"] / reps, 3),
                            "gbs": round(o["bytes"] / (o["ms"] / 1e3) / 1e9, 1) if o["ms"] else None}}
    del st.opt_state
    torch.cuda.empty_cache()
    return line


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings over the process group (the
    reported step time of a multi-GPU run is the slowest rank's)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def replica_throughput(tokens_per_step, steps, world, max_ms):
    """Whole-job tokens/s of `world` replicas that each ran `steps` steps."""
    return world * tokens_per_step * steps / (max_ms / 1e3)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def measure(w, args, rank, world, dev, barrier, *, optimizer=False, e2e=True):
    """Time one workload: an untraced timed region (the headline), then a
    second pass with the per-launch trace attached (the per-kernel breakdown
    and the roofline site), then the end-to-end host-buffer pass.  With
    --dp (and several ranks) every step is a data-parallel step: the ranks'
    gradients are summed over NCCL, overlapped with the backward."""
    import torch

    from decoder_only_gpt_b200 import binding as B
    from decoder_only_gpt_b200 import runtime as R

    wr = w.replace(seed=w.seed + 100 * rank)  # each rank its own batch
    cfg = B.config_from_workload(w)
    st = R.TrainStep(cfg, device=str(dev))
    bits = synth.make_params(w, as_bits=True)
    st.load_params(bits)
    tok, tgt = synth.make_tokens(wr)
    st.set_batch(tok, tgt)
    N = w.batch * w.seq_len
    stream = torch.cuda.current_stream(dev)
    dps = None
    if args.dp and world > 1:
        from decoder_only_gpt_b200 import dp
        dps = dp.DataParallelStep(st)
    one_step = dps.run if dps is not None else st.step

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    code = st.status()
    if code != B.GPT_OK:
        raise SystemExit(f"device status after warm-up: {B.strerror(code)}")

    # the headline replays the step as one CUDA graph (the runtime's capture);
    # the data-parallel step (NCCL on a second stream) runs eagerly
    timed_step = one_step
    if not args.no_graph and dps is None:
        st.capture()
        for _ in range(2):
            st.replay()
        torch.cuda.synchronize()
        code = st.status()
        if code != B.GPT_OK:
            raise SystemExit(f"device status after graph warm-up: {B.strerror(code)}")
        timed_step = st.replay

    bus = None
    try:
        bus = torch.cuda.get_device_properties(dev).pci_bus_id
    except Exception:
        bus = None
    clocks = ClockSampler(bus if isinstance(bus, str) else None)

    # ---- timed region (device time, CUDA events on the launching stream; no trace) ----
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        timed_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    code = st.status()
    if code != B.GPT_OK:
        raise SystemExit(f"device status after timed steps: {B.strerror(code)}")
    eager_ms = None
    if timed_step is not one_step:  # the same steps launched one by one, for comparison
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            one_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        eager_ms = e0.elapsed_time(e1)

    # ---- the same steps again with every launch timed (breakdown only) ----
    per_step = 1200  # trace records per step: ~500 launches, ~650 with the FP8 quantizers
    trace = B.Trace(capacity=per_step * args.steps + 16)
    barrier()
    torch.cuda.synchronize()
    trace.attach()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        one_step()
    t1.record(stream)
    torch.cuda.synchronize()
    B.Trace.detach()
    traced_ms = t0.elapsed_time(t1)
    stats, dropped = trace.summary()
    records = trace.records(per_step * args.steps + 16)
    trace.close()
    sites = gemm_sites(records, w, args.steps)

    # ---- end to end through the public host-buffer call ----
    e2e_ms = None
    if e2e and dps is not None:
        # the data-parallel step through its public call: this step's tokens
        # and targets from pinned host memory, the global loss back to the host
        ht = torch.from_numpy(tok.ravel().copy()).pin_memory()
        hy = torch.from_numpy(tgt.ravel().copy()).pin_memory()
        hl = torch.zeros(1, dtype=torch.float32).pin_memory()
        barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            st.tokens.copy_(ht, non_blocking=True)
            st.targets.copy_(hy, non_blocking=True)
            dps.run()
            hl.copy_(dps.global_loss, non_blocking=True)
            stream.synchronize()
            assert math.isfinite(float(hl[0]))
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = f0.elapsed_time(f1)
    elif e2e:
        ht = torch.from_numpy(tok.ravel().copy()).pin_memory()
        hy = torch.from_numpy(tgt.ravel().copy()).pin_memory()
        hl = torch.zeros(1, dtype=torch.float32).pin_memory()
        B.train_step_host(cfg, ht, hy, st.params, st.workspace, st.grads, hl, stream=stream.cuda_stream)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            B.train_step_host(cfg, ht, hy, st.params, st.workspace, st.grads, hl,
                              stream=stream.cuda_stream)
            stream.synchronize()  # the loss is read on the host every step
            assert math.isfinite(float(hl[0]))
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = f0.elapsed_time(f1)

    # ---- optimizer step (AdamW + Muon), timed on its own: not part of the
    # fwd+bwd metric; single-GPU runs only ----
    optim = None
    if optimizer and world == 1 and cfg.dtype == B.GPT_BF16:
        optim = time_optimizer(B, st, stream)

    out = dict(w=w, N=N, ms=ms, eager_ms=eager_ms, traced_ms=traced_ms, e2e_ms=e2e_ms, stats=stats,
               dropped=dropped,
               sites=sites, clk=clk, optim=optim, bits=bits)
    del st
    torch.cuda.empty_cache()
    return out


def summarize(m, args, world, peaks):
    """Throughput, MFU and the per-kernel breakdown of one measured workload."""
    w, N, ms = m["w"], m["N"], m["ms"]
    tok_s = replica_throughput(N, args.steps, world, ms)
    fpt = flops_per_token(w)
    stats = m["stats"]
    g = stats["gemm"]
    gemm_tf = g["flops"] / (g["ms"] / 1e3) / 1e12 if g["ms"] > 0 else 0.0
    peak_tf = peaks["bf16_tflops_sustained"]
    breakdown = {k: {"ms_per_step": round(v["ms"] / args.steps, 3),
                     "launches_per_step": v["launches"] // max(args.steps, 1),
                     **({"tflops": round(v["flops"] / (v["ms"] / 1e3) / 1e12, 1)} if v["flops"] and v["ms"] else {}),
                     **({"gbs": round(v["bytes"] / (v["ms"] / 1e3) / 1e9, 1)} if not v["flops"] and v["ms"] else {})}
                 for k, v in stats.items() if v["launches"]}
    kernels_per_step = sum(s["kernels"] for s in stats.values()) / max(args.steps, 1)
    return dict(tok_s=tok_s, fpt=fpt, gemm_tf=gemm_tf, peak_tf=peak_tf, breakdown=breakdown,
                kernels_per_step=kernels_per_step,
                mfu=round(tok_s / world * fpt / NOMINAL_BF16_FLOPS, 4),
                mfu_measured=round(tok_s / world * fpt / (peak_tf * 1e12), 4))


# nominal dense bf16 tensor-core peak of one B200 (public datasheet figure)
NOMINAL_BF16_FLOPS = 2.25e15


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    w = bench_workload(args)
    main_m = measure(w, args, rank, world, dev, barrier, optimizer=not args.no_optimizer)
    # the other depth the metric names, after the headline one (default runs)
    second = None
    if not args.no_second and args.workload == WORKLOAD and not (args.layers or args.batch or args.kv_heads
                                                                  or args.window or args.fp8
                                                                  or args.variants):
        second = measure(synth.workload(SECOND_WORKLOAD), args, rank, world, dev, barrier, e2e=False)

    ms, e2e_ms = main_m["ms"], main_m["e2e_ms"]
    ms2 = second["ms"] if second else 0.0
    if world > 1:
        ms, e2e_ms, ms2 = max_over_ranks([ms, e2e_ms, ms2], dev)
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    main_m["ms"], main_m["e2e_ms"] = ms, e2e_ms
    if second:
        second["ms"] = ms2

    peaks = load_peaks()
    s = summarize(main_m, args, world, peaks)
    N = main_m["N"]

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only) ----
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        setup = oracle_sample_setup(w, main_m["bits"])
        n = sample_tokens(setup)
        secs = time_oracle(setup)
        cpu = {"value": round(n / secs, 3), "unit": "tokens/s",
               "cores": cpu_cores(), "kind": "oracle",
               "sample": f"fp64 NumPy oracle fwd+bwd of the {w.name} model on the first "
                         f"{n} positions of one sequence ({secs:.1f} s)"}

    line = {
        "metric": METRIC,
        "value": round(s["tok_s"], 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 + e4m3 block projections (forward and data gradients)" if w.fp8 else "bf16",
        "data": "synthetic (Zipf(1.1) token ids, seeded N(0,0.02) bf16 weights)",
        "config": {"workload": workload_desc(w), "global_batch": w.batch * world,
                   "seq_len": w.seq_len, "tokens_per_step": N * world,
                   "parallelism": (f"data parallel x{world} (gradients summed over NCCL, overlapped with "
                                   "the backward)" if args.dp else f"replicas only x{world}")
                                  if world > 1 else "single GPU",
                   "l2": "no flush: every step moves tens of GB, far above the 126 MB L2",
                   "timing": ("headline untraced, the step replayed as one CUDA graph "
                              "(eager_ms_per_step: the same steps launched one by one); "
                              if main_m["eager_ms"] is not None else "headline untraced; ")
                             + "breakdown and roofline from a second, traced pass of eager launches"},
        "mfu": s["mfu"],
        "mfu_peak": "nominal dense bf16 2.25 PFLOP/s",
        "mfu_vs_measured_sustained": s["mfu_measured"],
        "flops_per_token": s["fpt"],
        "roofline": roofline(main_m["sites"], w, s["gemm_tf"], s["peak_tf"], peaks),
        "kernel_breakdown": s["breakdown"],
        "gemm_sites": main_m["sites"],
        "eager_ms_per_step": (round(main_m["eager_ms"] / args.steps, 3)
                              if main_m["eager_ms"] is not None else None),
        "traced_ms_per_step": round(main_m["traced_ms"] / args.steps, 3),
        "gpu_launches": int(round(s["kernels_per_step"] * args.steps)),
        "trace_dropped": main_m["dropped"],
        "e2e": {"value": round(replica_throughput(N, args.steps, world, e2e_ms), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": 2 * N * 4, "d2h_bytes_per_step": 4},
        "clocks": main_m["clk"],
        "cpu_baseline": cpu,
    }
    if main_m["optim"] is not None:
        line["optimizer"] = main_m["optim"]
    if second:
        s2 = summarize(second, args, world, peaks)
        w2 = second["w"]
        line[w2.name] = {"workload": workload_desc(w2), "value": round(s2["tok_s"], 1), "unit": "tokens/s",
                         "ms_per_step": round(ms2 / args.steps, 3), "mfu": s2["mfu"],
                         "mfu_vs_measured_sustained": s2["mfu_measured"], "flops_per_token": s2["fpt"],
                         "kernel_breakdown": s2["breakdown"], "gemm_sites": second["sites"],
                         "gpu_launches": int(round(s2["kernels_per_step"] * args.steps)),
                         "clocks": second["clk"]}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------
def run_reference(args, rank):
    if rank != 0:
        return
    w = bench_workload(args)
    setup = oracle_sample_setup(w, target_s=8.0)
    n = sample_tokens(setup)
    if args.warmup > 0:
        time_oracle(setup)  # one untimed sample
    secs = time_oracle(setup, steps=args.steps)
    value = n * args.steps / secs
    sample = (f"fp64 NumPy oracle fwd+bwd of the {w.name} model on the first {n} "
              f"positions of one sequence per step")
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "tokens/s",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (Zipf(1.1) token ids, seeded N(0,0.02) bf16 weights)",
        "config": {"workload": workload_desc(w), "global_batch": w.batch, "seq_len": w.seq_len,
                   "tokens_per_step": n, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cpu_cores(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD, choices=list(synth.WORKLOADS))
    ap.add_argument("--no-optimizer", action="store_true",
                    help="skip the separate timing of the optimizer step")
    ap.add_argument("--dp", action="store_true",
                    help="with several ranks: data-parallel steps (the ranks' gradients summed over "
                         "NCCL, overlapped with the backward) instead of independent replicas")
    ap.add_argument("--no-second", action="store_true",
                    help="skip the depth-12 measurement that default runs add")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip timing the CPU oracle sample")
    ap.add_argument("--no-graph", action="store_true",
                    help="time eager launches instead of the step replayed as one CUDA graph")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the workload's layer count (profiling captures on a smaller "
                         "case; the line then reports that model)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (profiling captures on a smaller "
                         "case; the line then reports that batch)")
    ap.add_argument("--kv-heads", type=int, default=0,
                    help="grouped-query attention with this many key/value heads (a model "
                         "variant; the line then reports it)")
    ap.add_argument("--window", type=int, default=0,
                    help="sliding attention window in positions (a model variant)")
    ap.add_argument("--fp8", action="store_true",
                    help="e4m3 operands in the forward block projections (a variant)")
    ap.add_argument("--variants", action="store_true",
                    help="block variants: value embeddings on every other layer, residual "
                         "scaling, smear and backout (a model variant)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
