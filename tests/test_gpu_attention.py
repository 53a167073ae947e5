"""The attention kernel (C-ABI test hook) against the oracle's attention on
the same bf16 inputs: bidirectional canvas passes and causal context chunks,
grouped-query packing, split-KV merges, ragged key and query counts."""

import numpy as np
import pytest
import torch

from oracle.model import attention as oracle_attention

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,nq,L0,Hq,Hkv,hd,causal,splits", [
    (1, 256, 64, 8, 8, 32, 0, 1), (1, 256, 64, 8, 8, 32, 0, 5), (1, 64, 0, 8, 8, 32, 1, 1),
    (1, 44, 256, 8, 8, 32, 1, 3), (2, 256, 77, 16, 8, 176, 0, 4), (1, 256, 1024, 16, 8, 176, 0, 5),
    (1, 256, 256, 16, 8, 176, 1, 4), (1, 200, 0, 16, 8, 176, 1, 1),
    (1, 256, 300, 8, 8, 32, 0, 8), (1, 256, 2048, 16, 8, 176, 0, 5), (2, 256, 77, 8, 8, 32, 0, 4)])
def test_attention_matches_oracle(B, nq, L0, Hq, Hkv, hd, causal, splits):
    import discrete_diffusion_moe_b200 as dg
    rng = np.random.default_rng(nq + L0 + hd + splits)
    c_max = L0 + nq + 5
    q = torch.from_numpy(rng.standard_normal((B * nq, Hq * hd)).astype(np.float32)).to(torch.bfloat16)
    k = torch.from_numpy(rng.standard_normal((B, Hkv, c_max, hd)).astype(np.float32)).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((B, Hkv, c_max, hd)).astype(np.float32)).to(torch.bfloat16)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    out = torch.zeros(B * nq, Hq * hd, dtype=torch.bfloat16, device="cuda")
    po = torch.zeros(max(splits, 1) * B * Hq * nq * hd, device="cuda")
    pml = torch.zeros(max(splits, 1) * B * Hq * nq * 2, device="cuda")
    dg.check(dg.lib.dg_test_attention(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), out.data_ptr(), B, nq, L0,
                                      c_max, Hq, Hkv, hd, causal, splits, po.data_ptr(), pml.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream))
    got = out.float().cpu().numpy().reshape(B, nq, Hq, hd)
    qn = q.double().numpy().reshape(B, nq, Hq, hd)
    kn = k.double().numpy().transpose(0, 2, 1, 3)[:, :L0 + nq]
    vn = v.double().numpy().transpose(0, 2, 1, 3)[:, :L0 + nq]
    for b in range(B):
        ref = oracle_attention(qn[b], kn[b], vn[b], np.arange(L0, L0 + nq), np.arange(L0 + nq), bool(causal))
        # P is carried as bf16 hi + lo parts, so the only sizeable error is the bf16
        # rounding of the output: at most one bf16 ulp (2^-7 relative) per element
        err = np.abs(got[b] - ref)
        bound = 2.0 ** -7 * np.abs(ref) + 2.0 ** -20 * np.abs(ref).max()
        assert np.all(err <= bound), (b, float((err / np.maximum(bound, 1e-30)).max()))
