"""Host side of the Python binding (no GPU): a round's per-position and
per-canvas results are views of one contiguous block (one device-to-host copy
reads them all), each view 16-byte aligned, disjoint from the others and the
exact buffer the C ABI receives."""

import numpy as np
import pytest
import torch


@pytest.mark.parametrize("batch", [1, 3, 16])
def test_step_outputs_pack_results_in_one_block(batch):
    import discrete_diffusion_moe_b200 as dg
    cfg = dg.model_config(n_layers=2, d_model=256, n_q_heads=8, n_kv_heads=8, head_dim=32, n_experts=16,
                          top_k=2, d_ff=512, vocab=4096)
    out = dg.StepOutputs(cfg, batch, device="cpu")
    names = ["argmax", "sample", "entropy", "pmax", "lock", "mean_entropy", "stop", "final_round"]
    base = out.packed.data_ptr()
    spans = []
    for name in names:
        t = getattr(out, name)
        lead = (batch,) if name in ("mean_entropy", "stop", "final_round") else (batch, 256)
        assert tuple(t.shape) == lead, name
        off = t.data_ptr() - base
        assert off % 16 == 0 and t.is_contiguous(), name
        assert getattr(out.s, name) == t.data_ptr(), name  # what the C ABI writes to
        spans.append((off, off + t.numel() * t.element_size(), name))
    spans.sort()
    for (a0, a1, na), (b0, b1, nb) in zip(spans, spans[1:]):
        assert a1 <= b0, (na, nb)
    assert spans[-1][1] <= out.packed.numel()
    assert out.packed.numel() - spans[-1][1] < 16  # no more than the last view's padding
    # writing one view leaves the others untouched
    out.entropy.fill_(1.5)
    assert torch.all(out.pmax == 0) and torch.all(out.argmax == 0) and torch.all(out.mean_entropy == 0)
    # optional outputs stay off the packed block and are null in the ABI struct unless asked for
    assert out.logits is None and out.s.logits is None and out.s.hidden is None
    full = dg.StepOutputs(cfg, batch, logits=True, routing=True, hidden=True, device="cpu")
    assert tuple(full.logits.shape) == (batch, 256, 4096)
    assert tuple(full.route_idx.shape) == (2, batch * 256, 2)
    assert tuple(full.route_logits.shape) == (2, batch * 256, 16)
    assert tuple(full.hidden.shape) == (3, batch * 256, 256)
    assert tuple(full.hidden_attn.shape) == (2, batch * 256, 256)
    assert full.s.hidden_attn == full.hidden_attn.data_ptr()
    assert full.s.logits == full.logits.data_ptr()
