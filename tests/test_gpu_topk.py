"""The top-k form of the expected embedding (the high-batch variant of the
self-conditioning input), the kernel on its own through its C-ABI test hook,
against oracle.sampler.expected_embedding_topk on crafted bf16 logits: random
rows, rows of few distinct values (many ids tie at the K-th largest, so the
lowest ids among them decide), rows of one value (every id ties), K = 1 (the
argmax row) and K = V."""

import numpy as np
import pytest
import torch

from oracle import sampler as OS
from oracle.numerics import bf16_round

pytestmark = pytest.mark.gpu


class _Emb:
    """The embedding rows the oracle's function reads."""

    def __init__(self, rows):
        self.rows = rows

        class _C:
            d_model = rows.shape[1]
        self.cfg = _C()

    def emb_rows(self, toks):
        return self.rows[np.asarray(toks)]


def _logits(kind, T, V, rng):
    if kind == "random":
        return rng.standard_normal((T, V)) * 2.0
    if kind == "few_values":      # 12 distinct values: hundreds of ids tie at every one
        return rng.integers(0, 12, size=(T, V)).astype(np.float64) * 0.25
    if kind == "equal":           # every id ties
        return np.full((T, V), 0.5)
    if kind == "peaked":          # a few large logits on a flat floor, ties inside the floor
        x = np.zeros((T, V))
        for t in range(T):
            x[t, rng.choice(V, 40, replace=False)] = rng.standard_normal(40) + 6.0
        return x
    raise ValueError(kind)


@pytest.mark.parametrize("kind,V,K,d,T", [
    ("random", 262144, 64, 256, 6), ("random", 8192, 64, 2816, 4), ("random", 4096, 1024, 256, 20),
    ("random", 4096, 1, 256, 9), ("few_values", 4096, 64, 256, 7), ("few_values", 16384, 1000, 512, 5),
    ("equal", 4096, 77, 256, 3), ("equal", 1024, 1024, 128, 2), ("peaked", 262144, 64, 256, 4),
    ("peaked", 8192, 300, 256, 5), ("random", 256, 256, 64, 3)])
def test_topk_expected_embedding_matches_oracle(kind, V, K, d, T):
    import discrete_diffusion_moe_b200 as dg
    rng = np.random.default_rng(V + K + T)
    lb = bf16_round(_logits(kind, T, V, rng))
    E = bf16_round(rng.standard_normal((V, d)) * 0.05)
    g_l = torch.from_numpy(lb.astype(np.float32)).to(torch.bfloat16).cuda()
    g_e = torch.from_numpy(E.astype(np.float32)).to(torch.bfloat16).cuda()
    out = torch.full((T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    dg.check(dg.lib.dg_test_expected_embedding_topk(g_l.data_ptr(), V, K, g_e.data_ptr(), d, T, out.data_ptr(),
                                                    torch.cuda.current_stream().cuda_stream))
    got = out.float().cpu().numpy().astype(np.float64)
    want, _ = OS.expected_embedding_topk(lb.astype(np.float32), _Emb(E), K)
    # one bf16 ulp of e, plus the rounding of each bf16 p_v (2^-8 of the largest |e|)
    tol = 2.0 ** -7 * np.abs(want) + 2.0 ** -8 * np.abs(want).max(axis=1, keepdims=True)
    bad = np.abs(got - want) > tol
    # (where ids tie at the K-th value, taking other ids than the lowest would
    # change the sum by whole embedding rows)
    assert not bad.any(), (int(bad.sum()), float(np.abs(got - want).max()))


def test_topk_hook_refuses_bad_arguments():
    import discrete_diffusion_moe_b200 as dg
    x = torch.zeros(512, dtype=torch.bfloat16, device="cuda")
    for V, K, d in ((300, 4, 64), (512, 0, 64), (512, 2000, 64), (512, 4, 100)):
        assert dg.lib.dg_test_expected_embedding_topk(x.data_ptr(), V, K, x.data_ptr(), d, 1, x.data_ptr(),
                                                      None) == dg.DG_ERR_INVALID_ARG
