"""A finished block appended to the context in the same pass as the next
canvas round (dg_denoise_step_append, dg_decode_block_ex): against the
oracle's definition (the causal encode of the block, then the round) -- the
appended keys and values of every layer, the logits, the decisions end to
end (tests/parity.py's free-running accounting) and the canvas update on the
GPU's statistics; and dg_decode_block_ex with a pending block equal, bit for
bit, to the same rounds called one by one."""

import numpy as np
import pytest
import torch

import synth
import oracle
from oracle import decode as OD
from oracle import sampler as OS
from parity import (TINY, LOGIT_REL, ROUTER_REL, Report, check_context_kv, compare_decisions, gpu_sampler,
                    rel_err, tf_update)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,C,self_cond", [(1, 40, False), (2, 77, True), (2, 64, False)])
def test_append_round_matches_encode_then_round(B, C, self_cond):
    """The appended block's keys and values of every layer against the
    oracle's causal encode; the round end to end against the oracle's
    definition (encode, then the round), which continues with the GPU's expert
    choices and compares its own routing decision by decision (the accounting
    of tests/parity.py: a routing flip at a near-tie moves its token's logits
    at O(1)); the canvas update on the GPU's statistics (strict)."""
    import discrete_diffusion_moe_b200 as dg
    cfg_d = TINY
    cfg = dg.model_config(**cfg_d, self_cond=self_cond)
    ocfg = oracle.ModelConfig(**cfg_d, self_cond=self_cond)
    W = oracle.Weights(ocfg, seed=0)
    model = dg.Model(cfg, B, seed=0, prefill_tokens=B * 512)
    c_max = C + 512
    ctx = synth.context_tokens(B, C, 1234, cfg.vocab)
    gkv = dg.KVCache(cfg, B, c_max)
    model.encode(gkv, torch.from_numpy(ctx.astype(np.int32)).cuda())
    okv = oracle.KVCache(ocfg, B, c_max)
    OD.encode_context(ocfg, W, okv, ctx)
    block = synth.context_tokens(B, 256, 99, cfg.vocab).astype(np.int32)   # a finished block
    sc = OS.SamplerConfig(max_steps=4, seed=5)
    gs = gpu_sampler(dg, sc)
    gcv = dg.Canvas(cfg, B)
    model.canvas_init(gcv, 1, sc.seed)
    tokens_in = gcv.tokens.cpu().numpy()
    prev_in = gcv.prev_argmax.cpu().numpy()
    done_in = gcv.done.cpu().numpy().astype(bool)
    out = dg.StepOutputs(cfg, B, logits=True, routing=True)
    model.step_append(gkv, gcv, 1, 0, gs, torch.from_numpy(block).cuda(), out)
    model.check_device()
    assert gkv.length == C + 256
    T, V, k = B * 256, cfg.vocab, cfg.top_k
    gi = out.route_idx.cpu().numpy()                                 # [L, T, k], canvas rows
    gr = out.route_logits.cpu().numpy().astype(np.float64)
    state = OD.new_state(tokens_in, cfg.d_model)
    o = OD.denoise_step_append(ocfg, W, okv, state, sc, 1, 0, block, record_routing=True,
                               force_routing=lambda l: gi[l].reshape(B, 256, k))
    assert okv.length == C + 256
    rep = Report()
    # the appended block's keys and values (and the context's, unchanged)
    rec = []
    okv2 = oracle.KVCache(ocfg, B, c_max)
    OD.encode_context(ocfg, W, okv2, np.concatenate([ctx, block], axis=1), record=rec)
    check_context_kv(rep, ocfg, gkv, okv2, rec, B, C + 256)
    # the round, end to end
    for l, (idx, w, margin, _, rlog) in enumerate(o.routing):
        rlog = rlog.reshape(T, -1)
        rep.router_rel = max(rep.router_rel, rel_err(gr[l], rlog))
        assert rep.router_rel <= ROUTER_REL, (l, rep.router_rel)
        compare_decisions(f"route[{l}]", gi[l], idx.reshape(T, -1), margin.reshape(T), rep, upstream=True,
                          explain=2 * np.abs(gr[l] - rlog).max(axis=1))
    gl = out.logits.cpu().numpy().reshape(T, V)
    ol = o.logits.reshape(T, V)
    rep.logit_rel = rel_err(gl, ol)
    assert rep.logit_rel <= LOGIT_REL, rep.logit_rel
    d_l = np.abs(gl.astype(np.float64) - ol).max(axis=1)
    inv_t = float(OS.inv_temperature_f32(0, sc.max_steps, sc.t_start, sc.t_end))
    compare_decisions("argmax", out.argmax.cpu().numpy().reshape(T), o.argmax.reshape(T),
                      o.argmax_margin.reshape(T), rep, upstream=True, explain=2 * d_l)
    compare_decisions("sample", out.sample.cpu().numpy().reshape(T), o.sample.reshape(T),
                      o.sample_margin.reshape(T), rep, upstream=True, explain=2 * d_l * inv_t + 1e-5)
    # the canvas update on the GPU's statistics (strict)
    tf_update(rep, ocfg, sc, out, tokens_in, prev_in, done_in, gcv.tokens.cpu().numpy(), 1, 0)
    rep.compared_positions = T
    print(f"append round: {rep}")
    model.close()


def test_decode_block_with_pending_block_equals_its_rounds():
    import discrete_diffusion_moe_b200 as dg
    cfg = dg.model_config(**TINY)
    model = dg.Model(cfg, 1, seed=0, prefill_tokens=512)
    sc = dg.sampler_config(max_steps=3, stop_entropy=0.0, seed=11)
    ctx = torch.from_numpy(synth.context_tokens(1, 30, 1234, cfg.vocab).astype(np.int32)).cuda()
    pending = torch.from_numpy(synth.context_tokens(1, 256, 98, cfg.vocab).astype(np.int32)).cuda()
    # through dg_decode_block_ex: block 1 with block 0 pending, its own append deferred
    kv1 = dg.KVCache(cfg, 1, 30 + 3 * 256)
    model.encode(kv1, ctx)
    cv1 = dg.Canvas(cfg, 1)
    out1 = torch.zeros(1, 256, dtype=torch.int32, device="cuda")
    steps, rounds = model.decode_block(kv1, cv1, 1, sc, out1, pending=pending, defer_append=True)
    model.check_device()
    assert steps == [3] and rounds == 3 and kv1.length == 30 + 256
    # the same rounds one by one
    kv2 = dg.KVCache(cfg, 1, 30 + 3 * 256)
    model.encode(kv2, ctx)
    cv2 = dg.Canvas(cfg, 1)
    model.canvas_init(cv2, 1, 11)
    model.step_append(kv2, cv2, 1, 0, sc, pending)
    for s in (1, 2):
        model.step(kv2, cv2, 1, s, sc)
    model.check_device()
    assert kv2.length == 30 + 256
    assert torch.equal(cv2.tokens, out1)
    for l in range(cfg.n_layers):
        a1, b1 = kv1.layer_kv(l)
        a2, b2 = kv2.layer_kv(l)
        assert torch.equal(a1[:, :, :kv1.length], a2[:, :, :kv2.length])
        assert torch.equal(b1[:, :, :kv1.length], b2[:, :, :kv2.length])
    model.close()


def test_block_stats_count_the_routed_experts():
    """dg_block_stats: tokens per pass and, per layer, the distinct experts
    the router chose over the batch's canvas tokens, against the routing the
    same round records."""
    import discrete_diffusion_moe_b200 as dg
    cfg = dg.model_config(**TINY)
    model = dg.Model(cfg, 2, seed=0)
    sc = dg.sampler_config(max_steps=1, stop_entropy=0.0, seed=3)
    ctx = torch.from_numpy(synth.context_tokens(2, 40, 1234, cfg.vocab).astype(np.int32)).cuda()
    kv = dg.KVCache(cfg, 2, 40 + 256)
    model.encode(kv, ctx)
    cv = dg.Canvas(cfg, 2)
    out = torch.zeros(2, 256, dtype=torch.int32, device="cuda")
    steps, rounds = model.decode_block(kv, cv, 0, sc, out, defer_append=True)
    stats = model.last_block_stats
    assert rounds == 1 and steps == [1, 1] and kv.length == 40
    assert stats["tokens_per_pass"] == 512.0
    cv2 = dg.Canvas(cfg, 2)
    model.canvas_init(cv2, 0, 3)
    so = dg.StepOutputs(cfg, 2, routing=True)
    model.step(kv, cv2, 0, 0, sc, so)
    model.check_device()
    want = [float(torch.unique(so.route_idx[l]).numel()) for l in range(cfg.n_layers)]
    assert stats["distinct_experts"] == want, (stats["distinct_experts"], want)
    model.close()
