"""Data-parallel training step: one process per GPU, gradients summed over the
ranks with torch.distributed (NCCL on GPUs), the exchange overlapped with the
backward.

"ChatGPT'nizi 50 Dolara Nasil Egitirsiniz?", section "Dagitilmis Egitim":
every rank trains on its own slice of the batch and the ranks' gradients are
combined while the backward is still running (the page launches its
reductions asynchronously and waits for them only before the update).

Each rank runs gpt_forward_loss and gpt_backward_ex on its own batch with the
gradients scaled by 1/world, so that the sum over the ranks is the gradient
of the mean loss over all ranks' positions.  gpt_backward_ex records one CUDA
event per bucket of the flat gradient buffer when that bucket is final: the
lm_head first, then the layers from the last to the first, then the
embedding.  For each bucket, in that order, a communication stream waits on
its event and all-reduces (sums) the bucket, so the exchange of the last
layers overlaps the backward of the first ones; the compute stream waits for
the communication stream before anything reads the gradients.

All arithmetic of the step is the library's; this module only plans the
buckets and issues the collectives.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

from . import binding as B

Bucket = Tuple[int, int]  # (element offset, element count) in the flat gradient buffer


def bucket_plan(cfg: B.GptConfig) -> List[Bucket]:
    """Buckets in gpt_backward_ex's event order: [lm_head, layer 0 .. layer
    n_layer-1, wte]; a layer's bucket spans its four block matrices, which
    are contiguous in the parameter layout (with their alignment padding)."""
    def span(tensor, layer):
        off, r, c = B.param_offset(cfg, tensor, layer)
        return off, off + r * c

    buckets = [None] * (cfg.n_layer + 2)
    lo, hi = span(B.GPT_T_LM_HEAD, 0)
    buckets[0] = (lo, hi - lo)
    for l in range(cfg.n_layer):
        lo, _ = span(B.GPT_T_WQKV, l)
        _, hi = span(B.GPT_T_WDOWN, l)
        buckets[1 + l] = (lo, hi - lo)
    lo, hi = span(B.GPT_T_WTE, 0)
    buckets[cfg.n_layer + 1] = (lo, hi - lo)
    return buckets


def ready_order(n_layer: int) -> List[int]:
    """Bucket indices in the order their gradients become final."""
    return [0] + [1 + l for l in reversed(range(n_layer))] + [n_layer + 1]


def allreduce_buckets(flat, buckets: Sequence[Bucket], order: Sequence[int], group=None,
                      events=None, comm_stream=None) -> None:
    """Sum every bucket of the 1-D tensor `flat` over the ranks of `group`, in
    `order`.  With CUDA `events` (one per bucket), each all-reduce runs on
    `comm_stream` after that bucket's event; without, they run in turn on the
    current stream (the CPU / gloo path)."""
    import torch
    import torch.distributed as dist

    for i in order:
        off, n = buckets[i]
        view = flat[off:off + n]
        if events is None:
            dist.all_reduce(view, op=dist.ReduceOp.SUM, group=group)
            continue
        comm_stream.wait_event(events[i])
        with torch.cuda.stream(comm_stream):
            dist.all_reduce(view, op=dist.ReduceOp.SUM, group=group)


class DataParallelStep:
    """One data-parallel fwd+bwd step of a runtime.TrainStep on every rank."""

    def __init__(self, step, group=None):
        import torch
        import torch.distributed as dist

        self.step = step
        self.group = group
        self.world = dist.get_world_size(group)
        self.buckets = bucket_plan(step.cfg)
        self.order = ready_order(step.cfg.n_layer)
        self.comm = torch.cuda.Stream(device=step.device)
        self.events = [torch.cuda.Event() for _ in self.buckets]
        cur = torch.cuda.current_stream(step.device)
        for e in self.events:  # creates the events' handles
            e.record(cur)
        dtype = torch.bfloat16 if step.cfg.dtype == B.GPT_BF16 else torch.float32
        self.flat = step.grads.view(dtype)
        self.global_loss = torch.zeros(1, dtype=torch.float32, device=step.device)

    def run(self) -> None:
        """Forward, backward with the exchange overlapped, global mean loss in
        `global_loss`; on return the compute stream holds the summed gradients."""
        import torch
        import torch.distributed as dist

        st = self.step
        cur = torch.cuda.current_stream(st.device)
        st.forward()
        # this step's first all-reduce may not overwrite gradients that the
        # previous step's readers (on the compute stream) still use
        self.comm.wait_stream(cur)
        B.backward_ex(st.cfg, st.tokens, st.targets, st.params, st.workspace, st.grads,
                      grad_scale=1.0 / self.world, events=[e.cuda_event for e in self.events],
                      stream=cur.cuda_stream)
        allreduce_buckets(self.flat, self.buckets, self.order, self.group, self.events, self.comm)
        with torch.cuda.stream(self.comm):
            self.global_loss.copy_(st.loss)
            dist.all_reduce(self.global_loss, op=dist.ReduceOp.SUM, group=self.group)
            self.global_loss.div_(self.world)
        cur.wait_stream(self.comm)
