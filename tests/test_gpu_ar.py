"""The retained autoregressive mode (dg_ar_step) against the oracle's
(oracle.decode.ar_step): the same weights decoding one token at a time after
a causally encoded context; each step's input is the previous step's GPU
sample (given to both sides).  Logits within 2e-2; argmax and sample bit for
bit except at margins below 1e-3 or, along the chain, a capped number of
mismatches explained by the measured logit difference (tests/parity.py); the
appended keys and values against the oracle's."""

import numpy as np
import pytest
import torch

import synth
import oracle
from oracle import decode as OD
from parity import TINY, LOGIT_REL, Report, compare_decisions, gpu_layer_kv, rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg_d,B,C,steps", [(TINY, 2, 40, 6), (dict(TINY, n_layers=1, n_q_heads=8, n_kv_heads=2,
                                                                       head_dim=32), 3, 17, 4)])
def test_ar_steps_match_oracle(cfg_d, B, C, steps):
    import discrete_diffusion_moe_b200 as dg
    cfg = dg.model_config(**cfg_d)
    model = dg.Model(cfg, B, seed=0)
    ocfg = oracle.ModelConfig(**cfg_d)
    W = oracle.Weights(ocfg, seed=0)
    ctx = synth.context_tokens(B, C, 1234, cfg.vocab)
    gkv = dg.KVCache(cfg, B, C + steps + 256)
    model.encode(gkv, torch.from_numpy(ctx.astype(np.int32)).cuda())
    okv = oracle.KVCache(ocfg, B, C + steps + 256)
    OD.encode_context(ocfg, W, okv, ctx)
    rep = Report()
    tok = synth.context_tokens(B, 1, 77, cfg.vocab)[:, 0].astype(np.int32)
    amax = torch.zeros(B, dtype=torch.int32, device="cuda")
    samp = torch.zeros(B, dtype=torch.int32, device="cuda")
    logits = torch.zeros(B, cfg.vocab, device="cuda")
    T_ = 0.8
    for s in range(steps):
        model.ar_step(gkv, torch.from_numpy(tok).cuda(), T_, 1234, amax, samp, logits)
        model.check_device()
        ol, oa, osmp, s_gap, a_gap = OD.ar_step(ocfg, W, okv, tok, T_, 1234)
        assert gkv.length == okv.length == C + s + 1
        gl = logits.cpu().numpy()
        rep.logit_rel = max(rep.logit_rel, rel_err(gl, ol))
        assert rep.logit_rel <= LOGIT_REL, rep.logit_rel
        d_l = np.abs(gl.astype(np.float64) - ol).max(axis=1)
        inv_t = float(np.float32(1.0 / float(np.float32(T_))))
        compare_decisions("argmax", amax.cpu().numpy(), oa, a_gap, rep, upstream=True, explain=2 * d_l)
        compare_decisions("sample", samp.cpu().numpy(), osmp, s_gap, rep, upstream=True,
                          explain=2 * d_l * inv_t + 1e-5)
        tok = samp.cpu().numpy().astype(np.int32)       # the next input, on both sides
    for l in range(ocfg.n_layers):
        gk, gv = gpu_layer_kv(gkv, l, C + steps)
        for g_, o_ in ((gk, okv.k[l][:, :C + steps]), (gv, okv.v[l][:, :C + steps])):
            err = np.abs(g_ - o_)[:, C:].max() / max(np.abs(o_).max(), 1e-30)
            assert err < LOGIT_REL, f"layer {l}: appended keys / values differ by {err}"
    rep.compared_positions = B * steps
    print(f"AR steps: {rep}")
    model.close()
