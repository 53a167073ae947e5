"""The attention entry point that takes no scratch from its caller
(dg_attention_static_scratch) against the one that does (dg_test_attention):
same inputs, two calls in a row.  Both run the same kernel with the same key
splits in the same order, so the outputs must be identical bit for bit; each
is also checked against the oracle within the attention test's per-element
bound.  Kept in a file of its own, collected last, so that it runs both alone
in a fresh process and after every other GPU test has used the device."""

import numpy as np
import pytest
import torch

import attn_inputs
from oracle.model import attention as oracle_attention

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,nq,L0,Hq,Hkv,hd,causal,splits", [
    (1, 256, 1024, 16, 8, 176, 0, 5), (2, 256, 77, 8, 8, 32, 0, 4), (1, 44, 256, 8, 8, 32, 1, 3)])
def test_static_scratch_matches_caller_scratch(B, nq, L0, Hq, Hkv, hd, causal, splits):
    import discrete_diffusion_moe_b200 as dg
    dev, ref_in = attn_inputs.make(B, nq, L0, Hq, Hkv, hd, seed=nq + L0 + hd, pad=3)
    dq, dk, dv, c_max = dev["q"], dev["k"], dev["v"], dev["c_max"]
    stream = torch.cuda.current_stream().cuda_stream
    want = torch.zeros(B * nq, Hq * hd, dtype=torch.bfloat16, device="cuda")
    po = torch.zeros(splits * B * Hq * nq * hd, device="cuda")
    pml = torch.zeros(splits * B * Hq * nq * 2, device="cuda")
    dg.check(dg.lib.dg_test_attention(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), want.data_ptr(), B, nq, L0,
                                      c_max, Hq, Hkv, hd, causal, splits, po.data_ptr(), pml.data_ptr(), stream))
    want_np = want.float().cpu().numpy()
    ref = np.stack([oracle_attention(ref_in["q"][b], ref_in["k"][b], ref_in["v"][b], np.arange(L0, L0 + nq),
                                     np.arange(L0 + nq), bool(causal)) for b in range(B)]).reshape(B * nq, Hq * hd)
    ref_abs = np.stack([oracle_attention(ref_in["q"][b], ref_in["k"][b], np.abs(ref_in["v"][b]),
                                         np.arange(L0, L0 + nq), np.arange(L0 + nq), bool(causal))
                        for b in range(B)]).reshape(B * nq, Hq * hd)
    for call in range(2):
        out = torch.full((B * nq, Hq * hd), float("nan"), dtype=torch.bfloat16, device="cuda")
        dg.check(dg.lib.dg_attention_static_scratch(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), out.data_ptr(),
                                                    B, nq, L0, c_max, Hq, Hkv, hd, causal, splits, stream))
        got = out.float().cpu().numpy()
        assert np.all(np.isfinite(got)), call
        # same kernel, same splits, same merge order: identical bits
        assert torch.equal(out, want), (call, float(np.abs(got - want_np).max()))
        err = np.abs(got - ref)
        br = attn_inputs.bound(ref, L0 + nq, ref_abs)
        assert np.all(err <= br), (call, float((err / np.maximum(br, 1e-30)).max()))


def test_static_scratch_rejects_requests_beyond_its_array():
    import discrete_diffusion_moe_b200 as dg
    B, nq, L0, Hq, Hkv, hd, splits = 4, 256, 64, 16, 8, 176, 8   # 8*4*16*256*178*4 B > 16 MiB
    assert splits * B * Hq * nq * (hd + 2) * 4 > dg.DG_ATTN_STATIC_SCRATCH_BYTES
    dev, _ = attn_inputs.make(B, nq, L0, Hq, Hkv, hd, seed=7)
    dq, dk, dv, c_max = dev["q"], dev["k"], dev["v"], dev["c_max"]
    out = torch.zeros(B * nq, Hq * hd, dtype=torch.bfloat16, device="cuda")
    rc = dg.lib.dg_attention_static_scratch(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), out.data_ptr(), B, nq,
                                            L0, c_max, Hq, Hkv, hd, 0, splits,
                                            torch.cuda.current_stream().cuda_stream)
    assert rc == dg.DG_ERR_INVALID_ARG
    assert b"scratch array" in dg.lib.dg_last_error()
