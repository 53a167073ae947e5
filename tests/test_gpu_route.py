"""The routing launch (top-k, counting sort by expert, row gather): the slot
tables it leaves are a valid grouping of the (token, slot) pairs by expert, the
k gathered rows of a token are one and the same row, and the order in which
CTAs claim their runs of slots (atomics) never changes a result: two models
built from the same seed give bit-identical hidden states, routing and logits
round after round."""

import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

# 128 experts top-8 at a small width: many CTAs claim slots of the same expert
WIDE_ROUTER = dict(n_layers=2, d_model=256, n_q_heads=8, n_kv_heads=8, head_dim=32, n_experts=128, top_k=8,
                   d_ff=512, vocab=4096)


def _model(dg, batch, cfg_kw, seed=0):
    cfg = dg.model_config(**cfg_kw, self_cond=True)
    model = dg.Model(cfg, batch, seed=seed)
    kv = dg.KVCache(cfg, batch, 64 + 256 * 2)
    model.encode(kv, torch.from_numpy(synth.context_tokens(batch, 64, 3, cfg_kw["vocab"])).cuda())
    cv = dg.Canvas(cfg, batch)
    model.canvas_init(cv, 0, 11)
    return cfg, model, kv, cv


class _DeviceView:
    """A raw device range seen by torch (no copy)."""

    def __init__(self, ptr, count, typestr):
        self.__cuda_array_interface__ = {"shape": (count,), "typestr": typestr, "data": (ptr, False),
                                         "version": 3, "strides": None}


def _read_ws(dg, model, name, dtype, count):
    """The first `count` elements of a named workspace buffer, on the host."""
    ptr = ctypes.c_void_p()
    nbytes = ctypes.c_size_t()
    dg.check(dg.lib.dg_test_workspace_buffer(model.ctx, name.encode(), ctypes.byref(ptr), ctypes.byref(nbytes)))
    itemsize = torch.empty(0, dtype=dtype).element_size()
    assert count * itemsize <= nbytes.value, name
    torch.cuda.synchronize()
    typestr = {torch.int32: "<i4", torch.float32: "<f4", torch.bfloat16: "<i2"}[dtype]
    t = torch.as_tensor(_DeviceView(ptr.value, count, typestr), device="cuda").cpu()
    return t.view(torch.bfloat16) if dtype == torch.bfloat16 else t


@pytest.mark.parametrize("batch,cfg_kw", [(4, "TINY"), (2, "WIDE")])
def test_route_tables_group_pairs_by_expert(batch, cfg_kw):
    import discrete_diffusion_moe_b200 as dg
    from parity import TINY
    kw = TINY if cfg_kw == "TINY" else WIDE_ROUTER
    cfg, model, kv, cv = _model(dg, batch, kw)
    out = dg.StepOutputs(cfg, batch, routing=True)
    samp = dg.sampler_config(max_steps=4, seed=11, stop_entropy=0.0)
    model.step(kv, cv, 0, 0, samp, out)
    model.check_device()
    T, k, E, d = batch * 256, kw["top_k"], kw["n_experts"], kw["d_model"]
    P = T * k
    # tables of the last layer
    idx = out.route_idx[-1].reshape(P).cpu().numpy()
    off = _read_ws(dg, model, "off", torch.int32, E + 1).numpy()
    perm = _read_ws(dg, model, "perm", torch.int32, P).numpy()
    inv = _read_ws(dg, model, "inv", torch.int32, P).numpy()
    wperm = _read_ws(dg, model, "wperm", torch.float32, P).numpy()
    xperm = _read_ws(dg, model, "xperm", torch.bfloat16, P * d).reshape(P, d)
    w = out.route_w[-1].reshape(P).cpu().numpy()
    # offsets are the exclusive prefix sums of the expert counts
    counts = np.bincount(idx, minlength=E)
    assert off[0] == 0 and np.array_equal(np.diff(off), counts)
    # perm is a permutation, inv its inverse, each expert's slots hold its pairs
    assert np.array_equal(np.sort(perm), np.arange(P))
    assert np.array_equal(inv[perm], np.arange(P))
    for e in range(E):
        assert np.all(idx[perm[off[e]:off[e + 1]]] == e), e
    # routing weights follow the permutation exactly; the k slots of a token
    # hold the same gathered row, and different tokens' rows differ
    assert np.array_equal(wperm, w[perm])
    rows = xperm[torch.from_numpy(inv.reshape(T, k)).long()]        # [T, k, d]
    assert torch.equal(rows, rows[:, :1].expand(-1, k, -1))
    assert not torch.equal(rows[0, 0], rows[1, 0])


def test_results_do_not_depend_on_slot_claim_order():
    import discrete_diffusion_moe_b200 as dg
    batch = 4
    cfg, m1, kv1, cv1 = _model(dg, batch, WIDE_ROUTER)
    _, m2, kv2, cv2 = _model(dg, batch, WIDE_ROUTER)
    o1 = dg.StepOutputs(cfg, batch, logits=True, routing=True, hidden=True)
    o2 = dg.StepOutputs(cfg, batch, logits=True, routing=True, hidden=True)
    samp = dg.sampler_config(max_steps=4, seed=11, stop_entropy=0.0)
    for s in range(4):
        m1.step(kv1, cv1, 0, s, samp, o1)
        m2.step(kv2, cv2, 0, s, samp, o2, graph=True)
        torch.cuda.synchronize()
        for a, b in ((o1.hidden, o2.hidden), (o1.route_idx, o2.route_idx), (o1.route_w, o2.route_w),
                     (o1.logits, o2.logits), (o1.sample, o2.sample), (cv1.tokens, cv2.tokens),
                     (cv1.sc_state, cv2.sc_state)):
            assert torch.equal(a, b), s
    m1.check_device()
    m2.check_device()
