"""The training step captured as one CUDA graph (runtime.TrainStep.capture).

* a replay gives the eager step's loss and gradients bit for bit (the step is
  deterministic, and the graph holds the same launches);
* the graph reads its buffers in place: after set_batch with new tokens a
  replay gives the eager step of the new batch, bit for bit;
* the device status stays clean across replays.
"""
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
    return st, tok, tgt


@pytest.mark.parametrize("name,kw", [("story", dict(n_layer=2, batch=4)),
                                     ("story", dict(n_layer=2, batch=2, n_kv_head=2, window=100, fp8=True)),
                                     ("tiny", dict(ve_every=1, resid_lambdas=True, smear=True, backout=True))])
def test_graph_replay_matches_eager(mods, name, kw):
    import torch
    B, R = mods
    w = synth.workload(name, **kw)
    st, tok, tgt = _step(B, R, w)
    st.step()
    torch.cuda.synchronize()
    want_g, want_l = st.grads.clone(), st.loss.clone()
    st.grads.zero_()
    st.capture()
    st.grads.zero_()
    for _ in range(2):
        st.replay()
    torch.cuda.synchronize()
    assert st.status() == B.GPT_OK
    assert torch.equal(st.grads, want_g) and torch.equal(st.loss, want_l)

    # a new batch through the same graph
    tok2 = (tok + 7) % w.vocab
    st.set_batch(tok2, tgt)
    st.replay()
    torch.cuda.synchronize()
    ref, _, _ = _step(B, R, w)
    ref.set_batch(tok2, tgt)
    ref.step()
    torch.cuda.synchronize()
    assert torch.equal(st.grads, ref.grads) and torch.equal(st.loss, ref.loss)
    assert not torch.equal(st.grads, want_g)
