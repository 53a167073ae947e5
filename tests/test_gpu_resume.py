"""Checkpoint / resume of a block's decoding state: 48 rounds run straight
through must equal 20 rounds, the state saved to host memory (canvas tokens,
self-conditioning state, previous argmax, done flags, and the context KV
cache), a new context on a new workspace restored from it, and the remaining
28 rounds -- bit for bit, round by round.  The round loop whose state this
is: the laozijiushiniubi.cn article, section 四 (rounds of a block until the
stop rule or the 48-round budget)."""

import numpy as np
import pytest
import torch

from parity import TINY

pytestmark = pytest.mark.gpu

ROUNDS, SPLIT = 48, 20


def _setup(dg, cfg, seed_ctx=11):
    model = dg.Model(cfg, 2, seed=0, kind_std={2: 2.0})   # a peaked LM head: positions lock
    kv = dg.KVCache(cfg, 2, 96 + 256)
    g = torch.Generator().manual_seed(seed_ctx)
    toks = torch.randint(0, cfg.vocab, (2, 96), generator=g, dtype=torch.int32).cuda()
    model.encode(kv, toks)
    model.check_device()
    return model, kv


def _round(dg, cfg, model, kv, cv, s, samp):
    out = dg.StepOutputs(cfg, 2)
    model.step(kv, cv, 3, s, samp, out, graph=(s % 2 == 1))   # direct launches and graph replays
    model.check_device()
    return (cv.tokens.cpu().numpy().copy(), cv.sc_state.view(torch.int16).cpu().numpy().copy(),
            out.packed.cpu().numpy().copy())


def test_resume_equals_straight_run():
    import discrete_diffusion_moe_b200 as dg
    cfg = dg.model_config(**TINY, self_cond=True)
    samp = dg.sampler_config(lock_policy=dg.DG_LOCK_PROB, lock_threshold=0.9, max_steps=ROUNDS,
                             stop_entropy=0.0, seed=99)
    # straight run
    model, kv = _setup(dg, cfg)
    cv = dg.Canvas(cfg, 2)
    model.canvas_init(cv, 3, 99)
    straight = [_round(dg, cfg, model, kv, cv, s, samp) for s in range(ROUNDS)]
    model.close()

    # 20 rounds, save, drop everything on the device, restore into new objects, 28 rounds
    model, kv = _setup(dg, cfg)
    cv = dg.Canvas(cfg, 2)
    model.canvas_init(cv, 3, 99)
    resumed = [_round(dg, cfg, model, kv, cv, s, samp) for s in range(SPLIT)]
    saved = {name: getattr(cv, name).cpu().clone() for name in ("tokens", "sc_state", "prev_argmax", "done")}
    saved_kv = (kv.k.cpu().clone(), kv.v.cpu().clone(), kv.length, kv.s.c_max)
    model.close()
    del model, kv, cv
    torch.cuda.synchronize()

    model = dg.Model(cfg, 2, seed=0, kind_std={2: 2.0})
    kv = dg.KVCache(cfg, 2, saved_kv[3])
    kv.k.copy_(saved_kv[0])
    kv.v.copy_(saved_kv[1])
    kv.s.length = saved_kv[2]
    cv = dg.Canvas(cfg, 2)
    for name, t in saved.items():
        getattr(cv, name).copy_(t)
    resumed += [_round(dg, cfg, model, kv, cv, s, samp) for s in range(SPLIT, ROUNDS)]
    model.close()

    for s, (a, b) in enumerate(zip(straight, resumed)):
        for x, y, what in zip(a, b, ("canvas", "self-conditioning state", "round outputs")):
            assert np.array_equal(x, y), f"round {s}: {what} differs after resume"
    final_tokens = straight[-1][0]
    assert ((final_tokens >= 0) & (final_tokens < cfg.vocab)).all()
    # the rounds carried state: the canvas changed between rounds and the last
    # round (the budget) froze it
    assert not np.array_equal(straight[0][0], straight[1][0])
