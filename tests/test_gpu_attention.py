"""The tensor-core attention kernel (C-ABI test hook) against the oracle's
attention on the same bf16 inputs: bidirectional canvas passes and causal
context chunks, grouped-query packing, split-KV merges, ragged key and query
counts, every supported head dimension."""

import numpy as np
import pytest
import torch

import attn_inputs
from oracle.model import attention as oracle_attention

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,nq,L0,Hq,Hkv,hd,causal,splits", [
    (1, 256, 64, 8, 8, 32, 0, 1), (1, 256, 64, 8, 8, 32, 0, 5), (1, 64, 0, 8, 8, 32, 1, 1),
    (1, 44, 256, 8, 8, 32, 1, 3), (2, 256, 77, 16, 8, 176, 0, 4), (1, 256, 1024, 16, 8, 176, 0, 5),
    (1, 256, 256, 16, 8, 176, 1, 4), (1, 200, 0, 16, 8, 176, 1, 1),
    (1, 256, 300, 8, 8, 32, 0, 8), (1, 256, 2048, 16, 8, 176, 0, 5), (2, 256, 77, 8, 8, 32, 0, 4),
    (1, 256, 1024, 8, 4, 64, 0, 4), (1, 130, 70, 8, 2, 128, 1, 2), (3, 256, 1024, 16, 8, 176, 0, 1),
    (1, 1, 0, 16, 8, 176, 0, 1), (1, 256, 8000, 16, 8, 176, 0, 8),
    # passes after a context appended at a ragged offset, and appending passes
    # (the first 256 queries causal, the canvas's 256 bidirectional)
    (1, 256, 296, 8, 8, 32, 0, 8), (2, 256, 333, 8, 8, 32, 0, 4), (1, 256, 40, 8, 8, 32, 1, 5),
    (2, 256, 77, 8, 8, 32, 1, 4), (1, 512, 40, 8, 8, 32, 256, 4), (2, 512, 77, 8, 8, 32, 256, 2),
    (2, 512, 40, 8, 8, 32, 256, 2), (1, 512, 77, 16, 8, 176, 256, 4)])
@pytest.mark.parametrize("merge", ["cluster", "scratch"])
def test_attention_matches_oracle(B, nq, L0, Hq, Hkv, hd, causal, splits, merge):
    """merge: the key splits of a tile merge inside their thread-block cluster
    (the layers' form), or through caller scratch and a second kernel."""
    import discrete_diffusion_moe_b200 as dg
    if merge == "scratch" and splits == 1:
        pytest.skip("one split has nothing to merge")
    dev, ref = attn_inputs.make(B, nq, L0, Hq, Hkv, hd, seed=nq + L0 + hd + splits)
    out = torch.full((B * nq, Hq * hd), float("nan"), dtype=torch.bfloat16, device="cuda")
    po = torch.zeros(max(splits, 1) * B * Hq * nq * hd, device="cuda")
    pml = torch.zeros(max(splits, 1) * B * Hq * nq * 2, device="cuda")
    p_o, p_ml = (None, None) if merge == "cluster" else (po.data_ptr(), pml.data_ptr())
    dg.check(dg.lib.dg_test_attention(dev["q"].data_ptr(), dev["k"].data_ptr(), dev["v"].data_ptr(), out.data_ptr(),
                                      B, nq, L0, dev["c_max"], Hq, Hkv, hd, causal, splits, p_o, p_ml,
                                      torch.cuda.current_stream().cuda_stream))
    got = out.float().cpu().numpy().reshape(B, nq, Hq, hd)
    for b in range(B):
        pos, kpos = np.arange(L0, L0 + nq), np.arange(L0 + nq)
        n_c = nq if causal == 1 else causal   # queries [0, n_c) causal, the rest bidirectional
        want, want_abs = [], []
        for rows, cz in ((slice(0, n_c), True), (slice(n_c, nq), False)):
            if rows.start == rows.stop:
                continue
            want.append(oracle_attention(ref["q"][b][rows], ref["k"][b], ref["v"][b], pos[rows], kpos, cz))
            want_abs.append(oracle_attention(ref["q"][b][rows], ref["k"][b], np.abs(ref["v"][b]), pos[rows],
                                             kpos, cz))
        want, want_abs = np.concatenate(want), np.concatenate(want_abs)
        # bf16 rounding of the output, fp16 probabilities in the P V product and
        # fp32 accumulation noise (see attn_inputs.bound)
        err = np.abs(got[b] - want)
        bound = attn_inputs.bound(want, L0 + nq, want_abs)
        assert np.all(err <= bound), (b, float((err / np.maximum(bound, 1e-30)).max()))
