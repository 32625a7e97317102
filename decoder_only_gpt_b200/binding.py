"""ctypes binding of libgpt (include/gpt.h): argument marshalling only.

Every numeric step of the training step runs in the library's CUDA kernels;
this module loads the shared library, mirrors its structs and constants, and
moves bytes between NumPy / torch buffers and the flat parameter layout the
library defines.  If libgpt.so is missing or fails to load, importing the
functions raises: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgpt.so")

GPT_OK, GPT_EINVAL, GPT_EUNSUPPORTED, GPT_ECUDA, GPT_EDATA, GPT_ETIMEOUT, GPT_ENONFINITE = (
    0, -1, -2, -3, -4, -5, -6)
GPT_BF16, GPT_F32 = 0, 1
GPT_T_WTE, GPT_T_WQKV, GPT_T_WO, GPT_T_WUP, GPT_T_WDOWN, GPT_T_LM_HEAD = range(6)
GPT_T_VE, GPT_T_VE_GATE, GPT_T_LAMBDAS, GPT_T_SMEAR_GATE, GPT_T_SCALARS = range(6, 11)
GPT_W_STATUS, GPT_W_RESID, GPT_W_LSE, GPT_W_SORT_PERM, GPT_W_SORT_OFFS, GPT_W_ATTN_LSE = range(6)

_TENSOR_IDS = {"wqkv": GPT_T_WQKV, "wo": GPT_T_WO, "wup": GPT_T_WUP, "wdown": GPT_T_WDOWN}


class GptConfig(ctypes.Structure):
    _fields_ = [
        ("n_layer", ctypes.c_int32), ("d_model", ctypes.c_int32), ("n_head", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("vocab", ctypes.c_int32),
        ("seq_len", ctypes.c_int32), ("batch", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("qk_norm", ctypes.c_int32), ("n_kv_head", ctypes.c_int32), ("attn_window", ctypes.c_int32),
        ("fp8", ctypes.c_int32), ("ve_every", ctypes.c_int32), ("ve_gate_channels", ctypes.c_int32),
        ("resid_lambdas", ctypes.c_int32), ("smear", ctypes.c_int32), ("backout", ctypes.c_int32),
        ("rope_base", ctypes.c_float), ("norm_eps", ctypes.c_float),
        ("n_params", ctypes.c_int64), ("param_bytes", ctypes.c_uint64),
        ("workspace_bytes", ctypes.c_uint64),
    ]


class GptOptim(ctypes.Structure):
    """Mirror of gpt_optim (optimizer hyper-parameters of one step)."""
    _fields_ = [("adam_lr", ctypes.c_float), ("adam_beta1", ctypes.c_float),
                ("adam_beta2", ctypes.c_float), ("adam_eps", ctypes.c_float),
                ("adam_weight_decay", ctypes.c_float), ("muon_lr", ctypes.c_float),
                ("muon_momentum", ctypes.c_float), ("muon_nesterov", ctypes.c_int32),
                ("ns_steps", ctypes.c_int32), ("ns_coeffs", (ctypes.c_float * 3) * 8),
                ("step", ctypes.c_int64), ("normuon", ctypes.c_int32),
                ("normuon_beta2", ctypes.c_float)]

    def coeffs(self):
        return [tuple(float(x) for x in self.ns_coeffs[i]) for i in range(self.ns_steps)]

    def set_coeffs(self, triples):
        if len(triples) > 8:
            raise ValueError("at most 8 Newton-Schulz iterations")
        self.ns_steps = len(triples)
        for i, t in enumerate(triples):
            for j in range(3):
                self.ns_coeffs[i][j] = float(t[j])


class GptError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} ({code})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libgpt.so (raises OSError if it is absent: no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"{LIB_PATH} not built; run `python -m decoder_only_gpt_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64
        cfgp = ctypes.POINTER(GptConfig)
        L.gpt_config_init.argtypes = [cfgp]
        L.gpt_config_from_depth.argtypes = [cfgp, I, I, I, I]
        L.gpt_param_offset.argtypes = [cfgp, I, I, ctypes.POINTER(I64), ctypes.POINTER(I64),
                                       ctypes.POINTER(I64)]
        L.gpt_workspace_region.argtypes = [cfgp, I, I, ctypes.POINTER(U64), ctypes.POINTER(U64)]
        L.gpt_forward_loss.argtypes = [cfgp, P, P, P, P, P, P, P]
        L.gpt_backward.argtypes = [cfgp, P, P, P, P, P, I, P]
        L.gpt_backward_ex.argtypes = [cfgp, P, P, P, P, P, I, ctypes.c_float,
                                      ctypes.POINTER(ctypes.c_void_p), I, P]
        L.gpt_train_step_host.argtypes = [cfgp, P, P, P, P, P, I, P, P]
        L.gpt_status.argtypes = [P, P]
        L.gpt_strerror.argtypes = [I]
        L.gpt_strerror.restype = ctypes.c_char_p
        L.gpt_version.restype = ctypes.c_char_p
        optp = ctypes.POINTER(GptOptim)
        L.gpt_optim_defaults.argtypes = [optp]
        L.gpt_optim_state_bytes.argtypes = [cfgp, ctypes.POINTER(ctypes.c_size_t)]
        L.gpt_optim_init.argtypes = [cfgp, P, P, P]
        L.gpt_optim_step.argtypes = [cfgp, optp, P, P, P, P, P]
        L.gpt_wait_expiry_check.argtypes = [P, ctypes.c_int64, P]
        for f in ("gpt_config_init", "gpt_config_from_depth", "gpt_param_offset",
                  "gpt_workspace_region", "gpt_forward_loss", "gpt_backward",
                  "gpt_backward_ex", "gpt_train_step_host", "gpt_status", "gpt_optim_defaults",
                  "gpt_optim_state_bytes", "gpt_optim_init", "gpt_optim_step",
                  "gpt_wait_expiry_check"):
            getattr(L, f).restype = I
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().gpt_strerror(code).decode()


def _check(rc: int, what: str) -> None:
    if rc != GPT_OK:
        raise GptError(rc, what)


def make_config(n_layer, d_model, n_head, head_dim, d_ff, vocab, seq_len, batch,
                dtype="bf16", qk_norm=True, rope_base=10000.0, norm_eps=1e-6,
                n_kv_head=0, attn_window=0, fp8=False, check=True, ve_every=0, ve_gate_channels=0,
                resid_lambdas=False, smear=False, backout=False) -> GptConfig:
    c = GptConfig(n_layer, d_model, n_head, head_dim, d_ff, vocab, seq_len, batch,
                  GPT_BF16 if dtype == "bf16" else GPT_F32, int(bool(qk_norm)),
                  n_kv_head, attn_window, int(bool(fp8)), int(ve_every), int(ve_gate_channels),
                  int(bool(resid_lambdas)), int(bool(smear)), int(bool(backout)),
                  rope_base, norm_eps, 0, 0, 0)
    rc = lib().gpt_config_init(ctypes.byref(c))
    if check:
        _check(rc, "gpt_config_init")
    return c


def config_from_workload(w) -> GptConfig:
    """Config for a ``synth.Workload``-like object (shape fields + dtype)."""
    return make_config(w.n_layer, w.d_model, w.n_head, w.head_dim, w.d_ff, w.vocab, w.seq_len,
                       w.batch, w.dtype, w.qk_norm, w.rope_base, w.norm_eps,
                       getattr(w, "n_kv_head", 0), getattr(w, "window", 0), getattr(w, "fp8", False),
                       ve_every=getattr(w, "ve_every", 0),
                       ve_gate_channels=getattr(w, "ve_gate_channels", 0) if getattr(w, "ve_every", 0) else 0,
                       resid_lambdas=getattr(w, "resid_lambdas", False), smear=getattr(w, "smear", False),
                       backout=getattr(w, "backout", False))


def config_from_depth(depth: int, seq_len: int, batch: int, vocab: int) -> GptConfig:
    c = GptConfig()
    _check(lib().gpt_config_from_depth(ctypes.byref(c), depth, seq_len, batch, vocab),
           "gpt_config_from_depth")
    return c


def param_offset(cfg: GptConfig, tensor: int, layer: int = 0):
    off, r, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    _check(lib().gpt_param_offset(ctypes.byref(cfg), tensor, layer, ctypes.byref(off),
                                  ctypes.byref(r), ctypes.byref(c)), "gpt_param_offset")
    return off.value, r.value, c.value


def workspace_region(cfg: GptConfig, region: int, layer: int = 0):
    off, nb = ctypes.c_uint64(), ctypes.c_uint64()
    _check(lib().gpt_workspace_region(ctypes.byref(cfg), region, layer, ctypes.byref(off),
                                      ctypes.byref(nb)), "gpt_workspace_region")
    return off.value, nb.value


def tensor_slots(cfg: GptConfig):
    """(name, tensor id, layer) for every parameter tensor, in buffer order."""
    yield "wte", GPT_T_WTE, 0
    for l in range(cfg.n_layer):
        for short, tid in _TENSOR_IDS.items():
            yield f"layers.{l}.{short}", tid, l
    yield "lm_head", GPT_T_LM_HEAD, 0
    for l in range(cfg.n_layer):
        if cfg.ve_every > 0 and l % cfg.ve_every == cfg.ve_every - 1:
            yield f"ve.{l}", GPT_T_VE, l
            yield f"ve_gate.{l}", GPT_T_VE_GATE, l
    if cfg.resid_lambdas:
        yield "lambdas", GPT_T_LAMBDAS, 0
    if cfg.smear:
        yield "smear_gate", GPT_T_SMEAR_GATE, 0
    if cfg.smear or cfg.backout:
        yield "scalars", GPT_T_SCALARS, 0


def elem_dtype(cfg: GptConfig):
    return np.uint16 if cfg.dtype == GPT_BF16 else np.float32


def pack_params(cfg: GptConfig, arrays: Dict[str, np.ndarray]) -> np.ndarray:
    """Flat host buffer (uint16 bf16 bits or float32) in the library's layout."""
    dt = elem_dtype(cfg)
    flat = np.zeros(cfg.param_bytes // np.dtype(dt).itemsize, dtype=dt)
    for name, tid, layer in tensor_slots(cfg):
        off, r, c = param_offset(cfg, tid, layer)
        a = np.ascontiguousarray(arrays[name], dtype=dt)
        assert a.shape == (r, c), (name, a.shape, (r, c))
        flat[off:off + r * c] = a.ravel()
    return flat


def unpack_flat(cfg: GptConfig, flat: np.ndarray) -> Dict[str, np.ndarray]:
    """Split a flat buffer into named [rows, cols] views (same dtype)."""
    out = {}
    for name, tid, layer in tensor_slots(cfg):
        off, r, c = param_offset(cfg, tid, layer)
        out[name] = flat[off:off + r * c].reshape(r, c)
    return out


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def forward_loss(cfg, tokens, targets, params, workspace, loss, token_loss=None, stream=None):
    rc = lib().gpt_forward_loss(ctypes.byref(cfg), _ptr(tokens), _ptr(targets), _ptr(params),
                                _ptr(workspace), _ptr(loss), _ptr(token_loss), stream)
    _check(rc, "gpt_forward_loss")


def backward(cfg, tokens, targets, params, workspace, grads, accumulate=False, stream=None):
    rc = lib().gpt_backward(ctypes.byref(cfg), _ptr(tokens), _ptr(targets), _ptr(params),
                            _ptr(workspace), _ptr(grads), int(bool(accumulate)), stream)
    _check(rc, "gpt_backward")


def raw_backward_ex(cfg, tokens, targets, params, workspace, grads, accumulate=0, grad_scale=1.0,
                    events=None, stream=None):
    """gpt_backward_ex; `events` is a sequence of cudaEvent_t handles (ints) or None."""
    arr, n = None, 0
    if events is not None:
        n = len(events)
        arr = (ctypes.c_void_p * n)(*[ctypes.c_void_p(int(e)) for e in events])
    return lib().gpt_backward_ex(ctypes.byref(cfg), _ptr(tokens), _ptr(targets), _ptr(params),
                                 _ptr(workspace), _ptr(grads), int(accumulate), float(grad_scale),
                                 arr, n, stream)


def backward_ex(cfg, tokens, targets, params, workspace, grads, accumulate=False, grad_scale=1.0,
                events=None, stream=None):
    _check(raw_backward_ex(cfg, tokens, targets, params, workspace, grads, int(bool(accumulate)),
                           grad_scale, events, stream), "gpt_backward_ex")


def train_step_host(cfg, host_tokens, host_targets, params, workspace, grads, host_loss,
                    accumulate=False, stream=None):
    rc = lib().gpt_train_step_host(ctypes.byref(cfg), _ptr(host_tokens), _ptr(host_targets),
                                   _ptr(params), _ptr(workspace), _ptr(grads),
                                   int(bool(accumulate)), _ptr(host_loss), stream)
    _check(rc, "gpt_train_step_host")


def status(workspace, stream=None) -> int:
    return lib().gpt_status(_ptr(workspace), stream)


def raw_forward_loss(cfg, tokens, targets, params, workspace, loss, token_loss=None, stream=None):
    """As forward_loss, returning the code instead of raising."""
    return lib().gpt_forward_loss(ctypes.byref(cfg), _ptr(tokens), _ptr(targets), _ptr(params),
                                  _ptr(workspace), _ptr(loss), _ptr(token_loss), stream)


def raw_backward(cfg, tokens, targets, params, workspace, grads, accumulate=0, stream=None):
    return lib().gpt_backward(ctypes.byref(cfg), _ptr(tokens), _ptr(targets), _ptr(params),
                              _ptr(workspace), _ptr(grads), int(accumulate), stream)


# ---- tracing ----------------------------------------------------------------
GPT_K_NAMES = ["gemm", "attn_fwd", "attn_bwd", "norm", "qkv", "loss", "sort", "scatter", "other",
               "quant"]


class GptTraceStat(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int32), ("kernels", ctypes.c_int32), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


class GptTraceRecord(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("kernels", ctypes.c_int32), ("ms", ctypes.c_float),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


class Trace:
    """Per-launch CUDA-event trace of the library's kernels (see gpt_trace_* in gpt.h)."""

    def __init__(self, capacity: int):
        L = lib()
        L.gpt_trace_create.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]
        L.gpt_trace_attach.argtypes = [ctypes.c_void_p]
        L.gpt_trace_reset.argtypes = [ctypes.c_void_p]
        L.gpt_trace_summary.argtypes = [ctypes.c_void_p, ctypes.POINTER(GptTraceStat),
                                        ctypes.POINTER(ctypes.c_int32)]
        L.gpt_trace_destroy.argtypes = [ctypes.c_void_p]
        self._h = ctypes.c_void_p()
        _check(L.gpt_trace_create(ctypes.byref(self._h), capacity), "gpt_trace_create")

    def attach(self):
        _check(lib().gpt_trace_attach(self._h), "gpt_trace_attach")

    @staticmethod
    def detach():
        _check(lib().gpt_trace_attach(None), "gpt_trace_attach")

    def reset(self):
        _check(lib().gpt_trace_reset(self._h), "gpt_trace_reset")

    def summary(self):
        stats = (GptTraceStat * len(GPT_K_NAMES))()
        dropped = ctypes.c_int32()
        _check(lib().gpt_trace_summary(self._h, stats, ctypes.byref(dropped)), "gpt_trace_summary")
        out = {n: dict(launches=s.launches, kernels=s.kernels, ms=s.ms, flops=s.flops,
                       bytes=s.bytes) for n, s in zip(GPT_K_NAMES, stats)}
        return out, dropped.value

    def records(self, capacity: int):
        """Per-launch records in launch order: list of (kind name, kernels, ms, flops, bytes)."""
        L = lib()
        L.gpt_trace_records.argtypes = [ctypes.c_void_p, ctypes.POINTER(GptTraceRecord),
                                        ctypes.c_int, ctypes.POINTER(ctypes.c_int32)]
        buf = (GptTraceRecord * capacity)()
        n = ctypes.c_int32()
        _check(L.gpt_trace_records(self._h, buf, capacity, ctypes.byref(n)), "gpt_trace_records")
        return [(GPT_K_NAMES[r.kind], r.kernels, r.ms, r.flops, r.bytes) for r in buf[:n.value]]

    def close(self):
        if self._h:
            lib().gpt_trace_destroy(self._h)
            self._h = ctypes.c_void_p()


# ---- optimizer step ---------------------------------------------------------
def optim_defaults() -> GptOptim:
    o = GptOptim()
    _check(lib().gpt_optim_defaults(ctypes.byref(o)), "gpt_optim_defaults")
    return o


def optim_state_bytes(cfg: GptConfig) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().gpt_optim_state_bytes(ctypes.byref(cfg), ctypes.byref(n)), "gpt_optim_state_bytes")
    return int(n.value)


def optim_init(cfg, params, state, stream=None):
    _check(lib().gpt_optim_init(ctypes.byref(cfg), _ptr(params), _ptr(state), stream), "gpt_optim_init")


def raw_optim_step(cfg, opt, params, grads, state, workspace, stream=None) -> int:
    return lib().gpt_optim_step(ctypes.byref(cfg), ctypes.byref(opt) if opt is not None else None,
                                _ptr(params), _ptr(grads), _ptr(state), _ptr(workspace), stream)


def optim_step(cfg, opt, params, grads, state, workspace, stream=None):
    _check(raw_optim_step(cfg, opt, params, grads, state, workspace, stream), "gpt_optim_step")


def wait_expiry_check(workspace, limit_ns: int, stream=None) -> int:
    """Launch the bounded-wait expiry check; returns the launch code (the
    expiry itself is read with status())."""
    return lib().gpt_wait_expiry_check(_ptr(workspace), int(limit_ns), stream)
