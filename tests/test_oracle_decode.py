"""Invariants of the oracle's denoising step and decode loop (no GPU)."""

import numpy as np
import pytest

import synth
from oracle.model import ModelConfig, Weights, KVCache
from oracle.sampler import SamplerConfig, LOCK_PROB, LOCK_ENTROPY_CUMSUM
from oracle import decode as D


def _small(self_cond=False, lm_std=0.02):
    cfg = ModelConfig(n_layers=1, d_model=32, n_q_heads=4, n_kv_heads=2, head_dim=8, n_experts=4,
                      top_k=2, d_ff=16, vocab=64, self_cond=self_cond, canvas=16)
    W = Weights(cfg, seed=0, std={synth.KIND_LM: lm_std})
    kv = KVCache(cfg, 2, 8 + 16 * 3)
    D.encode_context(cfg, W, kv, synth.context_tokens(2, 8, 3, cfg.vocab))
    return cfg, W, kv


@pytest.mark.parametrize("policy,thr", [(LOCK_PROB, 0.9), (LOCK_ENTROPY_CUMSUM, 0.1)])
def test_locked_positions_keep_their_sample(policy, thr):
    cfg, W, kv = _small(lm_std=2.0)  # peaked logits so that some positions lock
    sc = SamplerConfig(lock_policy=policy, lock_threshold=thr, max_steps=8, stop_entropy=0.0,
                       seed=5)
    st = D.new_state(D.init_canvas(sc.seed, 0, 2, cfg.canvas, cfg.vocab), cfg.d_model)
    o = D.denoise_step(cfg, W, kv, st, sc, block=0, step=0)
    assert o.lock.any() and not o.lock.all()
    assert np.array_equal(o.tokens_out[o.lock], o.sample[o.lock])
    noise = np.stack([D.smp.renoise_tokens(sc.seed, b, 0, 0, cfg.canvas, cfg.vocab) for b in range(2)])
    assert np.array_equal(o.tokens_out[~o.lock], noise[~o.lock])


def test_final_step_outputs_argmax_and_freezes():
    cfg, W, kv = _small()
    sc = SamplerConfig(max_steps=2, stop_entropy=0.0, seed=1)
    st = D.new_state(D.init_canvas(sc.seed, 0, 2, cfg.canvas, cfg.vocab), cfg.d_model)
    o0 = D.denoise_step(cfg, W, kv, st, sc, 0, 0)
    assert not o0.final.any()
    o1 = D.denoise_step(cfg, W, kv, st, sc, 0, 1)
    assert o1.final.all() and st.done.all()
    assert np.array_equal(st.tokens, o1.argmax)
    frozen = st.tokens.copy()
    D.denoise_step(cfg, W, kv, st, sc, 0, 1)
    assert np.array_equal(st.tokens, frozen)


def test_stop_fires_at_threshold_step():
    cfg, W, kv = _small()
    sc = SamplerConfig(max_steps=6, stop_entropy=100.0, seed=1)  # every mean entropy is below
    toks, steps, outs = D.decode_block(cfg, W, kv, sc, block=0, batch=2)
    assert list(steps) == [1, 1] and len(outs) == 1 and outs[0].stop.all()
    assert np.array_equal(toks, outs[0].argmax)


def test_stable_argmax_rule_never_stops_at_step_zero():
    cfg, W, kv = _small()
    sc = SamplerConfig(max_steps=3, stop_entropy=100.0, stop_require_stable_argmax=True, seed=1)
    toks, steps, outs = D.decode_block(cfg, W, kv, sc, block=0, batch=1)
    assert not outs[0].stop.any()


def test_decode_deterministic_and_appends_block():
    cfg, W, kv = _small(self_cond=True)
    L0 = kv.length
    sc = SamplerConfig(max_steps=3, stop_entropy=0.0, seed=9)
    t1, s1, _ = D.decode_block(cfg, W, kv, sc, block=0, batch=2)
    assert kv.length == L0 + cfg.canvas
    cfg2, W2, kv2 = _small(self_cond=True)
    t2, s2, _ = D.decode_block(cfg2, W2, kv2, sc, block=0, batch=2)
    assert np.array_equal(t1, t2) and np.array_equal(s1, s2)
    assert np.array_equal(kv.k[0], kv2.k[0])


def test_self_conditioning_changes_later_steps_only():
    cfg_a, W_a, kv_a = _small(self_cond=True)
    cfg_b, W_b, kv_b = _small(self_cond=False)
    sc = SamplerConfig(max_steps=3, stop_entropy=0.0, seed=2)
    sa = D.new_state(D.init_canvas(sc.seed, 0, 2, 16, 64), 32)
    sb = D.new_state(D.init_canvas(sc.seed, 0, 2, 16, 64), 32)
    oa = D.denoise_step(cfg_a, W_a, kv_a, sa, sc, 0, 0)
    ob = D.denoise_step(cfg_b, W_b, kv_b, sb, sc, 0, 0)
    assert np.array_equal(oa.logits, ob.logits)  # e_prev = 0 at step 0
    assert np.abs(sa.sc).max() > 0
    oa = D.denoise_step(cfg_a, W_a, kv_a, sa, sc, 0, 1)
    ob = D.denoise_step(cfg_b, W_b, kv_b, sb, sc, 0, 1)
    assert not np.array_equal(oa.logits, ob.logits)


def test_canvas_init_uniform():
    toks = D.init_canvas(1234, 0, 4, 256, 4096)
    assert toks.shape == (4, 256) and toks.min() >= 0 and toks.max() < 4096
    # 1024 draws from 4096 ids: about 906 distinct (sd ~13)
    assert 850 < len(np.unique(toks)) < 960
