"""gpt_backward_ex and the data-parallel step on one B200.

* grad_scale: the backward is linear in the loss-gradient scale and a power
  of two scales every value exactly, so grad_scale = 1/2 gives exactly half
  of gpt_backward's gradients, bit for bit.
* grad_ready_events: a stream that waits for a bucket's event already sees
  that bucket's final values (lm_head first, then layer n_layer-1), and every
  event has been recorded once the step is done.
* DataParallelStep on a one-rank NCCL group runs the same events, stream and
  collective path as a multi-GPU run; its summed gradients are the plain
  step's and its global loss the local one.
"""
import os
import socket

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mods():
    from decoder_only_gpt_b200 import build
    build.build()
    from decoder_only_gpt_b200 import binding, runtime
    return binding, runtime


def _step(B, R, w):
    st = R.TrainStep(B.config_from_workload(w))
    st.load_params(synth.make_params(w, as_bits=True))
    tok, tgt = synth.make_tokens(w)
    st.set_batch(tok, tgt)
    return st


def test_grad_scale_half_is_exact(mods):
    import torch
    B, R = mods
    w = synth.workload("story", n_layer=2, batch=4)
    st = _step(B, R, w)
    st.step()
    want = st.grads.view(torch.bfloat16).float().cpu().numpy() * 0.5
    st.forward()
    B.backward_ex(st.cfg, st.tokens, st.targets, st.params, st.workspace, st.grads,
                  grad_scale=0.5, stream=st.stream)
    assert st.status() == B.GPT_OK
    got = st.grads.view(torch.bfloat16).float().cpu().numpy()
    assert np.array_equal(got, want)


def test_grad_ready_events_mark_final_buckets(mods):
    import torch
    B, R = mods
    from decoder_only_gpt_b200 import dp
    w = synth.workload("story", n_layer=3, batch=4)
    st = _step(B, R, w)
    cfg = st.cfg
    plan = dp.bucket_plan(cfg)
    cur = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    events = [torch.cuda.Event() for _ in plan]
    for e in events:
        e.record(cur)
    flat = st.grads.view(torch.bfloat16)
    snaps = {}
    st.forward()
    st.grads.fill_(0)
    B.backward_ex(cfg, st.tokens, st.targets, st.params, st.workspace, st.grads, grad_scale=1.0,
                  events=[e.cuda_event for e in events], stream=cur.cuda_stream)
    for i in (0, cfg.n_layer):  # lm_head, then the last layer
        off, n = plan[i]
        side.wait_event(events[i])
        with torch.cuda.stream(side):
            snaps[i] = flat[off:off + n].clone()
    torch.cuda.synchronize()
    assert st.status() == B.GPT_OK
    assert all(e.query() for e in events)
    for i, snap in snaps.items():
        off, n = plan[i]
        assert torch.equal(snap, flat[off:off + n]), i
        assert bool(snap.abs().max() > 0)


def test_backward_ex_rejects(mods):
    import torch
    B, R = mods
    w = synth.workload("story", n_layer=2, batch=2)
    st = _step(B, R, w)
    st.forward()
    ev = [torch.cuda.Event() for _ in range(st.cfg.n_layer + 1)]  # one too few
    for e in ev:
        e.record()
    rc = B.raw_backward_ex(st.cfg, st.tokens, st.targets, st.params, st.workspace, st.grads, 0, 1.0,
                           [e.cuda_event for e in ev], st.stream)
    assert rc == B.GPT_EINVAL
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        assert B.raw_backward_ex(st.cfg, st.tokens, st.targets, st.params, st.workspace, st.grads, 0,
                                 bad, None, st.stream) == B.GPT_EINVAL


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_data_parallel_step_single_rank(mods):
    import datetime

    import torch
    import torch.distributed as dist
    B, R = mods
    from decoder_only_gpt_b200 import dp
    w = synth.workload("story", n_layer=2, batch=4)
    ref = _step(B, R, w)
    ref.step()
    want = ref.grads.clone()
    st = _step(B, R, w)
    os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        step = dp.DataParallelStep(st)
        for _ in range(2):
            step.run()
        torch.cuda.synchronize()
        assert st.status() == B.GPT_OK
        assert torch.equal(st.grads, want)
        assert float(step.global_loss[0]) == float(ref.loss[0])
    finally:
        dist.destroy_process_group()
