"""Host-side tests of the C ABI (no GPU needed, no kernel launched).

The library is built if missing; every function declared in include/gpt.h
must be exported; configuration validation, the parameter layout and the
workspace regions are checked against the workload shapes; invalid arguments
are rejected before any CUDA call.
"""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def B():
    from decoder_only_gpt_b200 import build
    build.build()
    from decoder_only_gpt_b200 import binding
    return binding


def header_functions():
    src = open(os.path.join(ROOT, "include", "gpt.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gpt_[a-z_]+)\s*\(", src)))


def test_every_declared_function_is_exported(B):
    names = header_functions()
    assert "gpt_forward_loss" in names and "gpt_backward" in names and "gpt_config_init" in names
    lib = ctypes.CDLL(B.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_header_constants_match_binding(B):
    src = open(os.path.join(ROOT, "include", "gpt.h")).read()
    consts = dict(re.findall(r"#define (GPT_[A-Z0-9_]+) \(?(-?\d+)\)?", src))
    for k, v in consts.items():
        if hasattr(B, k):
            assert getattr(B, k) == int(v), k


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_config_derived_fields(B, name):
    w = synth.workload(name)
    c = B.config_from_workload(w)
    d, F, V, L = w.d_model, w.d_ff, w.vocab, w.n_layer
    assert c.n_params == 2 * V * d + L * (4 * d * d + 2 * F * d)
    assert c.n_params == sum(r * cc for _, (r, cc) in synth.param_shapes(w))
    esz = 2 if w.dtype == "bf16" else 4
    assert c.param_bytes >= c.n_params * esz
    assert c.param_bytes - c.n_params * esz < (2 + 4 * L) * 128 * esz
    assert c.workspace_bytes > 0 and c.workspace_bytes % 256 == 0


def test_depth_dial(B):
    for depth, d, H in [(4, 256, 2), (12, 768, 6), (24, 1536, 12)]:
        c = B.config_from_depth(depth, 2048, 16, 32768)
        assert (c.n_layer, c.d_model, c.n_head, c.head_dim, c.d_ff) == (depth, d, H, 128, 4 * d)
        assert c.dtype == B.GPT_BF16 and c.qk_norm == 1
    assert B.lib().gpt_config_from_depth(ctypes.byref(B.GptConfig()), 3, 64, 1, 100) == B.GPT_EINVAL


@pytest.mark.parametrize("kw,code", [
    (dict(d_model=100), "EINVAL"),              # != n_head * head_dim
    (dict(head_dim=32, d_model=128, n_head=4), "EUNSUPPORTED"),
    (dict(d_ff=100), "EUNSUPPORTED"),
    (dict(vocab=1), "EINVAL"),
    (dict(seq_len=0), "EINVAL"),
    (dict(batch=-1), "EINVAL"),
    (dict(n_kv_head=3), "EINVAL"),              # does not divide n_head
    (dict(n_kv_head=-2), "EINVAL"),
    (dict(attn_window=-1), "EINVAL"),
])
def test_config_rejects(B, kw, code):
    base = dict(n_layer=2, d_model=256, n_head=2, head_dim=128, d_ff=1024, vocab=4096,
                seq_len=64, batch=2)
    base.update(kw)
    c = B.make_config(**base, check=False)
    rc = B.lib().gpt_config_init(ctypes.byref(c))
    assert rc == getattr(B, "GPT_" + code)


def test_f32_config_rules(B):
    ok = B.make_config(2, 64, 4, 16, 256, 256, 64, 4, dtype="f32")
    assert ok.param_bytes % 4 == 0
    bad = B.make_config(2, 66, 2, 33, 256, 256, 64, 4, dtype="f32", check=False)
    assert B.lib().gpt_config_init(ctypes.byref(bad)) == B.GPT_EUNSUPPORTED


def test_gqa_and_window_config(B):
    # n_kv_head 0 means n_head; the q/k/v projection shrinks with n_kv_head
    c = B.make_config(2, 256, 4, 64, 1024, 4096, 128, 2)
    assert c.n_kv_head == 4 and c.attn_window == 0
    g = B.make_config(2, 256, 4, 64, 1024, 4096, 128, 2, n_kv_head=1, attn_window=48)
    assert g.n_kv_head == 1 and g.attn_window == 48
    d, F, V = 256, 1024, 4096
    assert g.n_params == 2 * V * d + 2 * ((d + 2 * 64) * d + d * d + 2 * F * d)
    assert B.param_offset(g, B.GPT_T_WQKV, 1)[1:] == (d + 2 * 64, d)
    assert g.param_bytes < c.param_bytes and g.workspace_bytes < c.workspace_bytes
    f = B.make_config(2, 64, 4, 16, 256, 256, 64, 4, dtype="f32", n_kv_head=2, attn_window=9)
    assert f.n_kv_head == 2


def test_fp8_config(B):
    c = B.make_config(2, 256, 4, 64, 1024, 4096, 128, 2)
    e = B.make_config(2, 256, 4, 64, 1024, 4096, 128, 2, fp8=True)
    assert e.fp8 == 1 and e.param_bytes == c.param_bytes
    # e4m3 weight codes (one byte per parameter) and one activation's codes
    assert e.workspace_bytes >= c.workspace_bytes + c.param_bytes // 2 + 256 * 1024
    bad = B.make_config(2, 64, 4, 16, 256, 256, 64, 4, dtype="f32", fp8=True, check=False)
    assert B.lib().gpt_config_init(ctypes.byref(bad)) == B.GPT_EUNSUPPORTED
    two = B.make_config(2, 256, 4, 64, 1024, 4096, 128, 2, check=False)
    two.fp8 = 2
    assert B.lib().gpt_config_init(ctypes.byref(two)) == B.GPT_EINVAL


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("story", {}), ("d24", {}),
                                     ("story", dict(n_kv_head=2, window=100)),
                                     ("tiny", dict(n_kv_head=1, window=3))])
def test_param_layout(B, name, kw):
    w = synth.workload(name, **kw)
    c = B.config_from_workload(w)
    esz = 2 if w.dtype == "bf16" else 4
    shapes = dict(synth.param_shapes(w))
    prev_end = 0
    for pname, tid, layer in B.tensor_slots(c):
        off, r, cc = B.param_offset(c, tid, layer)
        assert (r, cc) == shapes[pname]
        assert off % 128 == 0 and off >= prev_end
        prev_end = off + r * cc
    assert prev_end * esz <= c.param_bytes


def test_param_offset_rejects(B):
    c = B.config_from_workload(synth.workload("tiny"))
    o = ctypes.c_int64()
    assert B.lib().gpt_param_offset(ctypes.byref(c), 9, 0, ctypes.byref(o), ctypes.byref(o),
                                    ctypes.byref(o)) == B.GPT_EINVAL
    assert B.lib().gpt_param_offset(ctypes.byref(c), B.GPT_T_WO, 5, ctypes.byref(o),
                                    ctypes.byref(o), ctypes.byref(o)) == B.GPT_EINVAL


def test_workspace_regions_in_bounds(B):
    w = synth.workload("story")
    c = B.config_from_workload(w)
    for reg, layer in [(B.GPT_W_STATUS, 0), (B.GPT_W_RESID, 0), (B.GPT_W_LSE, 0),
                       (B.GPT_W_SORT_PERM, 0), (B.GPT_W_SORT_OFFS, 0), (B.GPT_W_ATTN_LSE, 2)]:
        off, nb = B.workspace_region(c, reg, layer)
        assert off % 256 == 0 and off + nb <= c.workspace_bytes
    N = w.batch * w.seq_len
    assert B.workspace_region(c, B.GPT_W_RESID)[1] == N * w.d_model * 4
    assert B.workspace_region(c, B.GPT_W_SORT_OFFS)[1] == (w.vocab + 1) * 4


def test_invalid_pointers_rejected_before_any_launch(B):
    c = B.config_from_workload(synth.workload("tiny"))
    a = 1 << 20  # fake, never dereferenced: validation fails first
    assert B.raw_forward_loss(c, None, a, a, a, a) == B.GPT_EINVAL
    assert B.raw_forward_loss(c, a + 4, a, a, a, a) == B.GPT_EINVAL      # misaligned tokens
    assert B.raw_forward_loss(c, a, a, a + 16, a, a) == B.GPT_EINVAL     # params not 256-aligned
    assert B.raw_backward(c, a, a, a, a, None) == B.GPT_EINVAL
    assert B.raw_backward(c, a, a, a, a, a, accumulate=2) == B.GPT_EINVAL
    stale = B.make_config(2, 64, 4, 16, 256, 256, 64, 4, dtype="f32")
    stale.batch = 8  # derived fields no longer match
    assert B.raw_forward_loss(stale, a, a, a, a, a) == B.GPT_EINVAL


def test_strerror(B):
    for code in range(0, -7, -1):
        assert B.strerror(code) and "unknown" not in B.strerror(code)
    assert "unknown" in B.strerror(-99)
    assert B.lib().gpt_version().startswith(b"libgpt")


def test_pack_unpack_roundtrip(B):
    w = synth.workload("tiny")
    c = B.config_from_workload(w)
    p = synth.make_params(w, as_bits=True)
    flat = B.pack_params(c, p)
    back = B.unpack_flat(c, flat)
    for k in p:
        assert np.array_equal(back[k], p[k])


# ---- optimizer step: argument checks (host side, no CUDA call is reached) ----
def test_optim_defaults_and_state_bytes():
    from decoder_only_gpt_b200 import binding as B
    o = B.optim_defaults()
    assert o.ns_steps == 2 and o.step == 1 and o.muon_nesterov == 1
    assert o.coeffs() == [(np.float32(8.156), np.float32(-22.483), np.float32(15.879)),
                          (np.float32(4.043), np.float32(-2.809), np.float32(0.5))]
    cfg = B.config_from_workload(synth.workload("story"))
    assert B.optim_state_bytes(cfg) == 3 * (cfg.param_bytes // 2) * 4


def test_optim_rejects():
    from decoder_only_gpt_b200 import binding as B
    cfg = B.config_from_workload(synth.workload("story"))
    o = B.optim_defaults()
    fake = 1 << 40  # 256-aligned, never dereferenced: every case fails before any launch
    assert B.raw_optim_step(cfg, None, fake, fake, fake, fake) == B.GPT_EINVAL
    assert B.raw_optim_step(cfg, o, None, fake, fake, fake) == B.GPT_EINVAL
    assert B.raw_optim_step(cfg, o, fake + 16, fake, fake, fake) == B.GPT_EINVAL
    for field, bad in (("ns_steps", 9), ("ns_steps", -1), ("step", 0), ("adam_beta1", 1.0),
                       ("adam_beta2", -0.5), ("muon_lr", float("nan")), ("muon_nesterov", 2)):
        o2 = B.optim_defaults()
        setattr(o2, field, bad)
        assert B.raw_optim_step(cfg, o2, fake, fake, fake, fake) == B.GPT_EINVAL, field
    o3 = B.optim_defaults()
    o3.ns_coeffs[1][2] = float("inf")
    assert B.raw_optim_step(cfg, o3, fake, fake, fake, fake) == B.GPT_EINVAL
    tiny = B.config_from_workload(synth.workload("tiny"))  # fp32 storage
    assert B.raw_optim_step(tiny, o, fake, fake, fake, fake) == B.GPT_EUNSUPPORTED


def test_wait_expiry_check_rejects():
    from decoder_only_gpt_b200 import binding as B
    fake = 1 << 40  # 256-aligned, never dereferenced: every case fails before any launch
    assert B.wait_expiry_check(None, 20_000_000) == B.GPT_EINVAL
    assert B.wait_expiry_check(fake + 16, 20_000_000) == B.GPT_EINVAL
    assert B.wait_expiry_check(fake, 10) == B.GPT_EINVAL
    assert B.wait_expiry_check(fake, 10**11) == B.GPT_EINVAL


def test_struct_mirrors_match_the_header(B, tmp_path):
    """The ctypes mirrors have the C layout: sizes and every field offset, as a
    C compiler lays the header's structs out."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    mirrors = {"gpt_config": B.GptConfig, "gpt_optim": B.GptOptim,
               "gpt_trace_stat": B.GptTraceStat, "gpt_trace_record": B.GptTraceRecord}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "gpt.h"', 'int main(void) {']
    for cname, py in mirrors.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ['  return 0;', '}']
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {tuple(l.split()[:2]): int(l.split()[2]) for l in out if l}
    for cname, py in mirrors.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)
