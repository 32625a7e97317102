"""Device buffers for one training step, owned through torch (memory and streams only).

``TrainStep`` allocates the flat parameter / gradient buffers, the workspace
and the loss outputs that libgpt needs, and calls the library's entry points
on the current torch stream.  All arithmetic happens inside libgpt.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import binding as B


def _bits_to_f64(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


class TrainStep:
    def __init__(self, cfg: B.GptConfig, device: str = "cuda"):
        if not torch.cuda.is_available():
            raise RuntimeError("libgpt needs a CUDA device (sm_100a); none is available")
        self.cfg = cfg
        self.device = torch.device(device)
        self.N = cfg.batch * cfg.seq_len
        u8 = dict(dtype=torch.uint8, device=self.device)
        self.params = torch.zeros(cfg.param_bytes, **u8)
        self.grads = torch.zeros(cfg.param_bytes, **u8)
        self.workspace = torch.zeros(cfg.workspace_bytes, **u8)
        self.loss = torch.zeros(1, dtype=torch.float32, device=self.device)
        self.token_loss = torch.zeros(self.N, dtype=torch.float32, device=self.device)
        self.tokens = torch.zeros(self.N, dtype=torch.int32, device=self.device)
        self.targets = torch.zeros(self.N, dtype=torch.int32, device=self.device)

    @property
    def stream(self):
        return torch.cuda.current_stream(self.device).cuda_stream

    # ---- parameters -----------------------------------------------------
    def load_params(self, arrays: Dict[str, np.ndarray]) -> None:
        flat = B.pack_params(self.cfg, arrays)
        self.params.copy_(torch.from_numpy(flat.view(np.uint8)))

    def set_batch(self, tokens: np.ndarray, targets: np.ndarray) -> None:
        self.tokens.copy_(torch.from_numpy(np.ascontiguousarray(tokens, dtype=np.int32).ravel()))
        self.targets.copy_(torch.from_numpy(np.ascontiguousarray(targets, dtype=np.int32).ravel()))

    # ---- the step ---------------------------------------------------------
    def forward(self, token_loss: bool = True) -> None:
        B.forward_loss(self.cfg, self.tokens, self.targets, self.params, self.workspace,
                       self.loss, self.token_loss if token_loss else None, self.stream)

    def backward(self, accumulate: bool = False) -> None:
        B.backward(self.cfg, self.tokens, self.targets, self.params, self.workspace, self.grads,
                   accumulate, self.stream)

    def step(self) -> None:
        self.forward()
        self.backward()

    # ---- the step as a CUDA graph --------------------------------------------
    def capture(self) -> None:
        """Record one forward + backward into a CUDA graph.  Every call of the
        step is stream-ordered device work (kernels, async copies and memsets;
        no host synchronisation, no allocation), so the whole step captures;
        ``replay`` then launches it as one graph, without the per-launch host
        work and gaps.  The graph reads the buffers in place: new tokens
        (``set_batch``) and parameters take effect on the next replay."""
        side = torch.cuda.Stream(self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(side):  # one eager step on the capture stream first
            self.step()
        torch.cuda.current_stream(self.device).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=side):
            self.step()

    def replay(self) -> None:
        self.graph.replay()

    def status(self) -> int:
        return B.status(self.workspace, self.stream)

    # ---- optimizer ----------------------------------------------------------
    def init_optimizer(self) -> None:
        """Allocate the optimizer state and copy the parameters into its fp32 master."""
        self.opt_state = torch.zeros(B.optim_state_bytes(self.cfg), dtype=torch.uint8,
                                     device=self.device)
        B.optim_init(self.cfg, self.params, self.opt_state, self.stream)

    def optimizer_step(self, opt: B.GptOptim) -> None:
        B.optim_step(self.cfg, opt, self.params, self.grads, self.opt_state, self.workspace,
                     self.stream)

    def optimizer_state(self):
        """(master, m, v) as host float32 arrays in the parameter buffer's layout."""
        st = self.opt_state.cpu().numpy().view(np.float32)
        pe = self.cfg.param_bytes // 2
        return st[:pe], st[pe:2 * pe], st[2 * pe:3 * pe]

    # ---- read-back --------------------------------------------------------
    def grads_f64(self) -> Dict[str, np.ndarray]:
        dt = B.elem_dtype(self.cfg)
        flat = self.grads.cpu().numpy().view(dt)
        return {k: _bits_to_f64(v) for k, v in B.unpack_flat(self.cfg, flat).items()}

    def grads_raw(self) -> np.ndarray:
        return self.grads.cpu().numpy().copy()

    def region(self, region: int, layer: int = 0) -> np.ndarray:
        off, nb = B.workspace_region(self.cfg, region, layer)
        return self.workspace[off:off + nb].cpu().numpy().copy()
