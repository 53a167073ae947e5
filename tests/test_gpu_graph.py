"""The CUDA-graph round (dg_denoise_step_graph) gives bit-identical results
to direct launches (dg_denoise_step), across rounds with different step
indices (the captured parameter node is updated per round), and through the
block loop."""

import numpy as np
import pytest
import torch

import synth
from parity import TINY

pytestmark = pytest.mark.gpu


def _setup(dg, self_cond):
    cfg = dg.model_config(**TINY, self_cond=self_cond)
    model = dg.Model(cfg, 2, seed=0)
    kv = dg.KVCache(cfg, 2, 100 + 256 * 2)
    model.encode(kv, torch.from_numpy(synth.context_tokens(2, 100, 5, TINY["vocab"])).cuda())
    cv = dg.Canvas(cfg, 2)
    model.canvas_init(cv, 0, 77)
    return cfg, model, kv, cv


@pytest.mark.parametrize("self_cond", [False, True])
def test_graph_round_matches_direct_launches(self_cond):
    import discrete_diffusion_moe_b200 as dg
    samp = dg.sampler_config(max_steps=5, seed=77, stop_entropy=0.0)
    cfg, m1, kv1, cv1 = _setup(dg, self_cond)
    _, m2, kv2, cv2 = _setup(dg, self_cond)
    o1 = dg.StepOutputs(cfg, 2, logits=True)
    o2 = dg.StepOutputs(cfg, 2, logits=True)
    for s in range(5):
        m1.step(kv1, cv1, 0, s, samp, o1)
        m2.step(kv2, cv2, 0, s, samp, o2, graph=True)
        torch.cuda.synchronize()
        for a, b in ((o1.logits, o2.logits), (o1.sample, o2.sample), (o1.entropy, o2.entropy),
                     (cv1.tokens, cv2.tokens), (cv1.sc_state, cv2.sc_state), (cv1.done, cv2.done)):
            assert torch.equal(a, b), s
    m1.check_device()
    m2.check_device()


def test_decode_block_runs_and_appends():
    import discrete_diffusion_moe_b200 as dg
    cfg, m, kv, cv = _setup(dg, True)
    out = torch.zeros(2, 256, dtype=torch.int32, device="cuda")
    L0 = kv.length
    steps, rounds = m.decode_block(kv, cv, 0, dg.sampler_config(max_steps=3, seed=9, stop_entropy=0.0), out)
    assert steps == [3, 3] and rounds == 3 and kv.length == L0 + 256
    assert torch.equal(out, cv.tokens)
    m.check_device()
