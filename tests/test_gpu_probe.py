"""The router-load probe (dg_router_probe): a layer's RMSNorm, router and
top-k on given hidden states N(0, 1), against the oracle's router on the same
states -- expert choices bit for bit except at routing margins below 1e-3."""

import numpy as np
import pytest
import torch

import synth
import oracle
from oracle import model as OM
from parity import FULL, TINY, Report, compare_decisions, rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg_d,layers,T", [(TINY, (0, 1), 256), (dict(FULL, n_layers=2), (1,), 256)])
def test_router_probe_matches_oracle(cfg_d, layers, T):
    import discrete_diffusion_moe_b200 as dg
    cfg = dg.model_config(**cfg_d)
    model = dg.Model(cfg, 1, seed=0)
    ocfg = oracle.ModelConfig(**cfg_d)
    W = oracle.Weights(ocfg, seed=0)
    rep = Report()
    x = synth.f32_tensor(T * cfg.d_model, 7, 905, 1.0).reshape(T, cfg.d_model)   # N(0, 1) hidden states
    xd = torch.from_numpy(x).cuda()
    idx = torch.zeros(T, cfg.top_k, dtype=torch.int32, device="cuda")
    for l in layers:
        model.router_probe(l, xd, idx)
        model.check_device()
        o_idx, _, margin, rlog = OM.router_block(ocfg, W.router(l), x.astype(np.float64).reshape(1, T, -1))
        compare_decisions(f"route[{l}]", idx.cpu().numpy(), o_idx.reshape(T, -1), margin.reshape(T), rep)
        counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=cfg.n_experts)
        assert counts.sum() == T * cfg.top_k
        print(f"layer {l}: {int((counts > 0).sum())} distinct experts, max load {counts.max()}, "
              f"mean {counts.mean():.1f}")
    assert rep.tf_decisions == T * len(layers)
    model.close()
