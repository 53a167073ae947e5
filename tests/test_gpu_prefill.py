"""Causal encode in long passes (a workspace sized for prefill passes of up
to N tokens, dg_context_create_ex): the context KV cache against the
oracle's causal encode of the same tokens, every layer (the near-tie rule of
tests/parity.py for context tokens whose routing margin is below 1e-3)."""

import numpy as np
import pytest
import torch

import synth
import oracle
from oracle import decode as OD
from parity import LAYER1, TINY, Report, check_context_kv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg_d,B,C,prefill", [(TINY, 1, 700, 1024), (TINY, 2, 333, 1024),
                                              (dict(LAYER1, vocab=4096), 1, 1500, 2048)])
def test_long_prefill_passes_match_oracle(cfg_d, B, C, prefill):
    import discrete_diffusion_moe_b200 as dg
    cfg = dg.model_config(**cfg_d)
    ocfg = oracle.ModelConfig(**cfg_d)
    W = oracle.Weights(ocfg, seed=0)
    ctx = synth.context_tokens(B, C, 1234, cfg.vocab)
    okv = oracle.KVCache(ocfg, B, C + 256)
    rec = []
    OD.encode_context(ocfg, W, okv, ctx, record=rec)
    rep = Report()
    model = dg.Model(cfg, B, seed=0, prefill_tokens=prefill)
    assert model.workspace.numel() > dg.lib.dg_workspace_bytes(cfg, B)
    gkv = dg.KVCache(cfg, B, C + 256)
    model.encode(gkv, torch.from_numpy(ctx.astype(np.int32)).cuda())
    model.check_device()
    assert gkv.length == C
    check_context_kv(rep, ocfg, gkv, okv, rec, B, C)
    print(f"prefill {prefill}: {rep}")
    model.close()
