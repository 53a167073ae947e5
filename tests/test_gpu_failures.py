"""Failure paths on the GPU, made without faulting it: a token id outside the
vocabulary reaching the device, a bounded wait that runs out, and calls after
each of them.  The device side only latches an error word (the token is
clamped, the wait gives up and its kernel returns); the host reads it with
dg_check_device_error, which reports and clears it, and the context stays
usable."""

import numpy as np
import pytest
import torch

from parity import TINY

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    import discrete_diffusion_moe_b200 as dg
    cfg = dg.model_config(**TINY)
    model = dg.Model(cfg, 1, seed=0)
    yield dg, cfg, model
    model.close()


def _step_ok(dg, cfg, model):
    kv = dg.KVCache(cfg, 1, 64 + 256)
    model.encode(kv, torch.arange(64, dtype=torch.int32, device="cuda").reshape(1, 64))
    cv = dg.Canvas(cfg, 1)
    model.canvas_init(cv, 0, 5)
    out = dg.StepOutputs(cfg, 1)
    model.step(kv, cv, 0, 0, dg.sampler_config(max_steps=4, seed=5), out)
    model.check_device()
    t = cv.tokens.cpu().numpy()
    assert ((t >= 0) & (t < cfg.vocab)).all()
    return out


def test_out_of_range_context_token_is_reported(tiny):
    dg, cfg, model = tiny
    kv = dg.KVCache(cfg, 1, 32 + 256)
    toks = torch.arange(32, dtype=torch.int32, device="cuda").reshape(1, 32)
    toks[0, 7] = cfg.vocab          # one past the last id
    model.encode(kv, toks)          # enqueued: the device clamps the id and latches the error
    with pytest.raises(dg.DgError) as e:
        model.check_device()
    assert e.value.status == dg.DG_ERR_BAD_TOKEN
    model.check_device()            # the error word was cleared
    _step_ok(dg, cfg, model)        # and the context still works


def test_negative_canvas_token_is_reported(tiny):
    dg, cfg, model = tiny
    kv = dg.KVCache(cfg, 1, 16 + 256)
    model.encode(kv, torch.arange(16, dtype=torch.int32, device="cuda").reshape(1, 16))
    model.check_device()
    cv = dg.Canvas(cfg, 1)
    model.canvas_init(cv, 0, 5)
    cv.tokens[0, 100] = -3
    model.step(kv, cv, 0, 0, dg.sampler_config(max_steps=4, seed=5))
    with pytest.raises(dg.DgError) as e:
        model.check_device()
    assert e.value.status == dg.DG_ERR_BAD_TOKEN
    _step_ok(dg, cfg, model)


def test_bounded_wait_that_runs_out_reports_timeout(tiny):
    dg, cfg, model = tiny
    stream = torch.cuda.current_stream().cuda_stream
    dg.check(dg.lib.dg_test_wait_timeout(model.ctx, 200_000_000, stream))   # 0.2 s
    with pytest.raises(dg.DgError) as e:
        model.check_device()
    assert e.value.status == dg.DG_ERR_TIMEOUT
    assert "bounded device wait" in dg.last_error()
    # the next calls run normally
    out = _step_ok(dg, cfg, model)
    assert np.isfinite(out.entropy.cpu().numpy()).all()
    assert dg.lib.dg_test_wait_timeout(model.ctx, 0, stream) == dg.DG_ERR_INVALID_ARG


def test_decode_block_surfaces_a_latched_error(tiny):
    # dg_decode_block reads the error word after every round: an error latched
    # before it (here a wait that ran out) ends the call with that status
    dg, cfg, model = tiny
    stream = torch.cuda.current_stream().cuda_stream
    kv = dg.KVCache(cfg, 1, 16 + 2 * 256)
    model.encode(kv, torch.arange(16, dtype=torch.int32, device="cuda").reshape(1, 16))
    model.check_device()
    cv = dg.Canvas(cfg, 1)
    dg.check(dg.lib.dg_test_wait_timeout(model.ctx, 100_000_000, stream))
    toks = torch.zeros(1, 256, dtype=torch.int32, device="cuda")
    with pytest.raises(dg.DgError) as e:
        model.decode_block(kv, cv, 0, dg.sampler_config(max_steps=4, seed=5), toks)
    assert e.value.status == dg.DG_ERR_TIMEOUT
    model.check_device()
    steps, rounds = model.decode_block(kv, cv, 0, dg.sampler_config(max_steps=4, seed=5), toks)
    assert 1 <= steps[0] <= 4 and rounds == steps[0]
