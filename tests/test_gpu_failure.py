"""The failure path shared by every pipeline kernel, exercised without any GPU
fault (needs a B200): a bounded mbarrier wait that nothing completes expires,
the kernel records GPT_ETIMEOUT in the status word and returns, and the same
context then runs a full training step normally.
"""
import math
import time

import pytest

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from decoder_only_gpt_b200 import build
    build.build()
    from decoder_only_gpt_b200 import binding
    return binding


def test_bounded_wait_expires_and_context_survives(B):
    import torch
    from decoder_only_gpt_b200 import runtime as R
    w = synth.workload("story")
    ts = R.TrainStep(B.config_from_workload(w))
    ts.load_params(synth.make_params(w, as_bits=True))
    tok, tgt = synth.make_tokens(w)
    ts.set_batch(tok, tgt)
    ts.step()
    assert ts.status() == B.GPT_OK
    t0 = time.monotonic()
    assert B.wait_expiry_check(ts.workspace, 20_000_000, ts.stream) == B.GPT_OK  # 20 ms limit
    code = ts.status()  # synchronises the stream
    elapsed = time.monotonic() - t0
    assert code == B.GPT_ETIMEOUT
    assert 0.015 <= elapsed < 5.0, elapsed
    # the same context: a full step clears the status word and runs normally
    ts.step()
    torch.cuda.synchronize()
    assert ts.status() == B.GPT_OK
    assert math.isfinite(float(ts.loss.item()))
