"""Data-parallel gradient exchange on CPU: world size 2 over gloo.

The bucket plan and the bucketed all-reduce of decoder_only_gpt_b200.dp are
the code the GPU path runs (there with NCCL and per-bucket CUDA events); here
each rank's gradient comes from the fp64 oracle on its half of the batch,
scaled by 1/world as gpt_backward_ex scales it.  The sum over the ranks must
equal the single-process gradient of the whole batch ("ChatGPT'nizi 50
Dolara Nasil Egitirsiniz?", section "Dagitilmis Egitim").
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("story", {}), ("d24", {}),
                                     ("story", dict(n_kv_head=2))])
def test_bucket_plan_covers_every_gradient_once(name, kw):
    from decoder_only_gpt_b200 import binding as B
    from decoder_only_gpt_b200 import dp
    w = synth.workload(name, **kw)
    cfg = B.config_from_workload(w)
    plan = dp.bucket_plan(cfg)
    assert len(plan) == cfg.n_layer + 2
    # every tensor lies in exactly the bucket the event order names for it
    owner = {"lm_head": 0, "wte": cfg.n_layer + 1}
    for tname, tid, layer in B.tensor_slots(cfg):
        off, r, c = B.param_offset(cfg, tid, layer)
        i = owner.get(tname, 1 + layer)
        lo, n = plan[i]
        assert lo <= off and off + r * c <= lo + n, tname
    # buckets are disjoint and inside the buffer
    spans = sorted(plan)
    for (a, na), (b, _) in zip(spans, spans[1:]):
        assert a + na <= b
    esz = 2 if cfg.dtype == B.GPT_BF16 else 4
    assert spans[-1][0] + spans[-1][1] <= cfg.param_bytes // esz
    # lm_head first, then the layers from the last, then the embedding
    assert dp.ready_order(cfg.n_layer) == [0] + list(range(cfg.n_layer, 0, -1)) + [cfg.n_layer + 1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from decoder_only_gpt_b200 import binding as B
    from decoder_only_gpt_b200 import dp
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    w = synth.workload("tiny")
    cfg = B.config_from_workload(w)
    params = synth.make_params(w)
    tok, tgt = synth.make_tokens(w)
    rows = list(range(rank * w.batch // world, (rank + 1) * w.batch // world))
    ocfg = oracle.from_workload(w)
    # this rank's gradient of its own mean loss, scaled by 1/world
    res = oracle.step(ocfg, params, tok[rows], tgt[rows])
    grads = {k: v / world for k, v in res.grads.items()}
    flat = torch.from_numpy(B.pack_params(cfg, grads).astype(np.float32))
    dp.allreduce_buckets(flat, dp.bucket_plan(cfg), dp.ready_order(cfg.n_layer))
    loss = torch.tensor([res.loss], dtype=torch.float64)
    dist.all_reduce(loss)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, flat.numpy().copy(), float(loss[0]) / world))


def test_two_gloo_ranks_sum_to_the_single_process_gradient():
    import oracle
    from decoder_only_gpt_b200 import binding as B
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    for _ in procs:
        r, flat, loss = q.get(timeout=300)
        out[r] = (flat, loss)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = synth.workload("tiny")
    cfg = B.config_from_workload(w)
    tok, tgt = synth.make_tokens(w)
    ref = oracle.step(oracle.from_workload(w), synth.make_params(w), tok, tgt)
    want = B.pack_params(cfg, ref.grads).astype(np.float32)
    for r in (0, 1):
        flat, loss = out[r]
        # both ranks hold the same sum: the whole batch's gradient (fp32 rounding)
        np.testing.assert_allclose(flat, want, rtol=2e-6, atol=1e-9)
        assert loss == pytest.approx(ref.loss, rel=1e-12)
    assert np.array_equal(out[0][0], out[1][0])
