"""Pins of the oracle's transformer pieces against closed forms, invariants
and independent formulations (no GPU)."""

import math

import numpy as np
import pytest
import torch

from oracle import model as M
from oracle.numerics import bf16_round, f32_round


# ---- rounding helpers -------------------------------------------------------

def test_bf16_round_ties_to_even():
    one = 1.0
    ulp = 2.0 ** -7  # bf16 spacing in [1, 2)
    assert bf16_round(one + ulp / 2) == one                 # tie, even stays
    assert bf16_round(one + 3 * ulp / 2) == one + 2 * ulp   # tie, odd rounds up
    assert bf16_round(one + ulp / 2 + 2.0 ** -30) == one + ulp
    assert bf16_round(-(one + 3 * ulp / 2)) == -(one + 2 * ulp)
    assert bf16_round(0.0) == 0.0


def test_bf16_round_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(bf16_round(x.astype(np.float64)), ref)


def test_f32_round():
    assert f32_round(1.0 + 2.0 ** -30) == 1.0
    assert f32_round(1.0 + 2.0 ** -23) == 1.0 + 2.0 ** -23


# ---- RMSNorm, RoPE, SwiGLU ----------------------------------------------------

def test_rmsnorm_closed_form():
    x = np.array([3.0, 4.0])
    rms = math.sqrt((9 + 16) / 2 + 1e-6)
    assert np.allclose(M.rmsnorm(x, 1e-6), x / rms, rtol=0, atol=1e-15)
    assert np.allclose(M.rmsnorm(x, 1e-6, gain=np.array([2.0, 0.5])), x / rms * [2.0, 0.5])


def test_rope_identity_at_position_zero():
    x = np.random.default_rng(1).standard_normal((3, 2, 8))
    assert np.allclose(M.rope(x, np.zeros(3), 10000.0), x, atol=0)


def test_rope_relative_position_and_norm():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 1, 16))
    k = rng.standard_normal((1, 1, 16))
    dots = []
    for shift in (0, 5, 1000):
        qr = M.rope(q, np.array([7 + shift]), 10000.0)
        kr = M.rope(k, np.array([3 + shift]), 10000.0)
        dots.append(float((qr * kr).sum()))
        assert np.isclose(np.linalg.norm(qr), np.linalg.norm(q))
    assert np.allclose(dots, dots[0], rtol=1e-10)


def test_rope_pairs_rotate_halves():
    # one pair (i, i + hd/2) at position p rotates by p * theta^(-2i/hd)
    hd, i, p, theta = 8, 1, 3, 10000.0
    x = np.zeros((1, 1, hd))
    x[0, 0, i] = 1.0
    ang = p * theta ** (-2.0 * i / hd)
    r = M.rope(x, np.array([p]), theta)[0, 0]
    assert np.isclose(r[i], math.cos(ang)) and np.isclose(r[i + hd // 2], math.sin(ang))
    assert np.allclose(np.delete(r, [i, i + hd // 2]), 0)


def test_silu_and_expert_closed_form():
    assert M.silu(np.array([0.0]))[0] == 0.0
    assert np.isclose(M.silu(np.array([1.0]))[0], 1 / (1 + math.exp(-1)))
    # one-hot weights pick single products: y = silu(a) * u * wd
    x = np.array([[1.0, 0.0]])
    wg = np.array([[2.0, 0.0]])
    wu = np.array([[0.5, 0.0]])
    wd = np.array([[1.0], [0.0]])
    want = bf16_round(2.0 / (1 + math.exp(-2.0)) * 0.5)
    assert np.isclose(M.expert_ffn(x, wg, wu, wd)[0, 0], want)


# ---- attention ----------------------------------------------------------------

def _attention_loop(q, k, v, q_pos, k_pos, causal):
    """A second formulation: per query and head, log-sum-exp weighted sum."""
    nq, Hq, hd = q.shape
    group = Hq // k.shape[1]
    out = np.zeros_like(q)
    for i in range(nq):
        for h in range(Hq):
            g = h // group
            keys = [j for j in range(k.shape[0]) if not causal or k_pos[j] <= q_pos[i]]
            s = [sum(q[i, h, t] * k[j, g, t] for t in range(hd)) / math.sqrt(hd) for j in keys]
            lse = max(s) + math.log(sum(math.exp(a - max(s)) for a in s))
            for j, a in zip(keys, s):
                out[i, h] += math.exp(a - lse) * v[j, g]
    return out


@pytest.mark.parametrize("causal", [False, True])
def test_attention_matches_second_formulation(causal):
    rng = np.random.default_rng(3)
    q = rng.standard_normal((5, 4, 6))
    k = rng.standard_normal((7, 2, 6))
    v = rng.standard_normal((7, 2, 6))
    q_pos = np.arange(2, 7)
    k_pos = np.arange(7)
    got = M.attention(q, k, v, q_pos, k_pos, causal)
    assert np.allclose(got, _attention_loop(q, k, v, q_pos, k_pos, causal), atol=1e-12)


def test_attention_permutation_equivariant_without_mask():
    rng = np.random.default_rng(4)
    n, ctx = 9, 4
    q = rng.standard_normal((n, 2, 8))
    kc = rng.standard_normal((n, 1, 8))
    vc = rng.standard_normal((n, 1, 8))
    kx = rng.standard_normal((ctx, 1, 8))
    vx = rng.standard_normal((ctx, 1, 8))
    perm = rng.permutation(n)
    pos = np.arange(ctx, ctx + n)
    kp = np.arange(ctx + n)
    a = M.attention(q, np.concatenate([kx, kc]), np.concatenate([vx, vc]), pos, kp, False)
    b = M.attention(q[perm], np.concatenate([kx, kc[perm]]), np.concatenate([vx, vc[perm]]),
                    pos, kp, False)
    assert np.allclose(a[perm], b, atol=1e-12)


def test_attention_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(5)
    k = np.repeat(rng.standard_normal((1, 1, 8)), 6, axis=0)
    v = rng.standard_normal((6, 1, 8))
    q = rng.standard_normal((3, 1, 8))
    out = M.attention(q, k, v, np.arange(3), np.arange(6), False)
    assert np.allclose(out, v.mean(axis=0, keepdims=True), atol=1e-12)


def test_causal_first_row_sees_only_itself():
    rng = np.random.default_rng(6)
    q, k, v = (rng.standard_normal((4, 1, 8)) for _ in range(3))
    out = M.attention(q, k, v, np.arange(4), np.arange(4), True)
    assert np.allclose(out[0], v[0])


# ---- routing / mixture of experts --------------------------------------------

def _toy_layer(rng, E, d, f):
    from oracle.numerics import f64_to_bf16_bits
    mk = lambda *s: bf16_round(rng.standard_normal(s) * 0.3)  # noqa: E731
    return {"wr": mk(E, d), "wg": f64_to_bf16_bits(mk(E, f, d)), "wu": f64_to_bf16_bits(mk(E, f, d)),
            "wd": f64_to_bf16_bits(mk(E, d, f))}


def test_moe_topk_all_equals_dense_softmax_mixture():
    from oracle.numerics import bf16_bits_to_f64 as dec
    rng = np.random.default_rng(7)
    E, d, f = 4, 8, 6
    layer = _toy_layer(rng, E, d, f)
    h = bf16_round(rng.standard_normal((5, d)))
    out, idx, w, _, _ = M.moe_ffn(h, layer, top_k=E)
    logits = f32_round(h @ layer["wr"].T)
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    dense = sum(p[:, [e]] * M.expert_ffn(h, dec(layer["wg"][e]), dec(layer["wu"][e]),
                                         dec(layer["wd"][e])) for e in range(E))
    assert np.allclose(out, dense, rtol=1e-6, atol=1e-6)


def test_moe_single_expert_is_plain_ffn():
    from oracle.numerics import bf16_bits_to_f64 as dec
    rng = np.random.default_rng(8)
    layer = _toy_layer(rng, 1, 8, 6)
    h = bf16_round(rng.standard_normal((3, 8)))
    out, idx, w, _, _ = M.moe_ffn(h, layer, top_k=1)
    assert np.all(idx == 0) and np.all(w == 1.0)
    assert np.array_equal(out, M.expert_ffn(h, dec(layer["wg"][0]), dec(layer["wu"][0]),
                                            dec(layer["wd"][0])))


def test_route_weights_sum_to_one_and_ties_go_low():
    wr = np.array([[1.0, 0.0], [1.0, 0.0], [0.5, 0.0], [1.0, 0.0]])  # experts 0, 1, 3 tie
    h = np.array([[1.0, 2.0]])
    idx, w, _ = M.route(h, wr, 2)
    assert list(idx[0]) == [0, 1]
    assert np.isclose(w.sum(), 1.0) and np.allclose(w, 0.5)
    rng = np.random.default_rng(9)
    idx, w, logits = M.route(rng.standard_normal((20, 8)), rng.standard_normal((16, 8)), 4)
    assert np.allclose(w.sum(1), 1.0, atol=1e-6)
    for t in range(20):
        assert set(idx[t]) == set(np.argsort(-logits[t], kind="stable")[:4])


# ---- one layer: how the pieces are wired ---------------------------------------

def _wired_layer(rng, d, Hq, Hkv, hd, E, f, zero_down=True):
    """A layer whose attention has a closed form: zero query and key weights
    make every score 0 (uniform attention over the visible keys); the value
    projection copies the first Hkv * hd features of the normed input; the
    output projection is the identity on the Hq * hd = d attention features."""
    from oracle.numerics import f64_to_bf16_bits
    assert Hq * hd == d
    wv = np.zeros((Hkv * hd, d))
    wv[:, :Hkv * hd] = np.eye(Hkv * hd)
    mk = lambda *s: bf16_round(rng.standard_normal(s) * 0.3)  # noqa: E731
    wd = np.zeros((E, d, f)) if zero_down else mk(E, d, f)
    return {"wq": np.zeros((Hq * hd, d)), "wk": np.zeros((Hkv * hd, d)), "wv": wv, "wo": np.eye(d),
            "wr": mk(E, d), "wg": f64_to_bf16_bits(mk(E, f, d)), "wu": f64_to_bf16_bits(mk(E, f, d)),
            "wd": f64_to_bf16_bits(wd)}


def _cfg(d, Hq, Hkv, hd, E, k, f):
    return M.ModelConfig(n_layers=1, d_model=d, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=hd, n_experts=E,
                         top_k=k, d_ff=f, vocab=256)


def _rms_bf16(x, eps=1e-6):
    return bf16_round(x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps))


def test_layer_with_zero_output_and_down_projections_keeps_the_stream():
    rng = np.random.default_rng(20)
    d, Hq, Hkv, hd, E, k, f = 16, 4, 2, 4, 4, 2, 8
    cfg = _cfg(d, Hq, Hkv, hd, E, k, f)
    lw = _wired_layer(rng, d, Hq, Hkv, hd, E, f)
    lw["wo"] = np.zeros((d, Hq * hd))
    x = f32_round(rng.standard_normal((1, 5, d)))
    kk = np.zeros((1, 8, Hkv, hd), np.float32)
    vv = np.zeros((1, 8, Hkv, hd), np.float32)
    y, _ = M.layer_forward(cfg, lw, x, kk, vv, 0, causal=True, append=True)
    assert np.array_equal(y, x)
    # the values written to the cache are the copied features of the normed rows
    h = _rms_bf16(x[0])
    assert np.array_equal(vv[0, :5].reshape(5, -1), h[:, :Hkv * hd].astype(np.float32))
    assert np.all(kk[0, :5] == 0) and np.all(vv[0, 5:] == 0)


@pytest.mark.parametrize("causal", [False, True])
def test_layer_attention_residual_in_closed_form(causal):
    # uniform attention: query i of head h returns the mean over its visible keys
    # of the copied features of kv head h // (Hq / Hkv); the identity output
    # projection puts head h at features [h * hd, (h + 1) * hd)
    rng = np.random.default_rng(21)
    d, Hq, Hkv, hd, E, k, f = 16, 4, 2, 4, 4, 2, 8
    G = Hq // Hkv
    cfg = _cfg(d, Hq, Hkv, hd, E, k, f)
    lw = _wired_layer(rng, d, Hq, Hkv, hd, E, f)
    L0, n = 3, 5
    x = f32_round(rng.standard_normal((1, n, d)))
    ctx_v = bf16_round(rng.standard_normal((L0, Hkv * hd)))
    kk = np.zeros((1, L0 + n, Hkv, hd), np.float32)
    vv = np.zeros((1, L0 + n, Hkv, hd), np.float32)
    vv[0, :L0] = ctx_v.reshape(L0, Hkv, hd)
    y, _ = M.layer_forward(cfg, lw, x, kk, vv, L0, causal=causal, append=False)
    vals = np.concatenate([ctx_v, _rms_bf16(x[0])[:, :Hkv * hd]])  # [L0 + n, Hkv * hd]
    want = np.empty((n, d))
    for i in range(n):
        vis = vals[:L0 + i + 1] if causal else vals
        mean = vis.mean(axis=0)
        for h in range(Hq):
            g = h // G
            want[i, h * hd:(h + 1) * hd] = mean[g * hd:(g + 1) * hd]
    want = f32_round(x[0] + bf16_round(want))
    assert np.array_equal(y[0], want)


def test_layer_moe_reads_the_stream_after_attention():
    # one expert (E = k = 1): the layer adds the SwiGLU FFN of the normed
    # stream AFTER the attention residual, not of the layer's input
    from oracle.numerics import bf16_bits_to_f64 as dec
    rng = np.random.default_rng(22)
    d, Hq, Hkv, hd, E, k, f = 16, 4, 4, 4, 1, 1, 8
    cfg = _cfg(d, Hq, Hkv, hd, E, k, f)
    lw = _wired_layer(rng, d, Hq, Hkv, hd, E, f, zero_down=False)
    n = 4
    x = f32_round(rng.standard_normal((1, n, d)))
    kk = np.zeros((1, n, Hkv, hd), np.float32)
    vv = np.zeros((1, n, Hkv, hd), np.float32)
    y, (idx, w, _, _) = M.layer_forward(cfg, lw, x, kk, vv, 0, causal=False, append=False)
    x1 = f32_round(x[0] + bf16_round(np.broadcast_to(_rms_bf16(x[0]).mean(axis=0), (n, d))))
    h2 = _rms_bf16(x1)
    a = h2 @ dec(lw["wg"][0]).T
    ffn = f32_round(bf16_round(a / (1.0 + np.exp(-a)) * (h2 @ dec(lw["wu"][0]).T)) @ dec(lw["wd"][0]).T)
    assert np.all(idx == 0) and np.all(w == 1.0)
    assert np.array_equal(y[0], f32_round(x1 + ffn))
    # a layer that fed the MoE with its input instead would differ
    h_in = _rms_bf16(x[0])
    a_in = h_in @ dec(lw["wg"][0]).T
    ffn_in = f32_round(bf16_round(a_in / (1.0 + np.exp(-a_in)) * (h_in @ dec(lw["wu"][0]).T)) @ dec(lw["wd"][0]).T)
    assert not np.array_equal(y[0], f32_round(x1 + ffn_in))


# ---- final norm + LM head --------------------------------------------------------

class _LmRows:
    """Stands in for the weights: vocabulary rows of a given matrix."""

    def __init__(self, rows):
        self.rows = rows

    def lm_chunk(self, v0, n):
        return self.rows[v0:v0 + n]


def test_lm_logits_closed_form_and_chunking():
    rng = np.random.default_rng(23)
    d, V = 16, 40
    cfg = M.ModelConfig(n_layers=1, d_model=d, n_q_heads=4, n_kv_heads=4, head_dim=4, n_experts=4, top_k=2,
                        d_ff=8, vocab=V)
    rows = np.zeros((V, d))
    rows[:d] = np.eye(d)          # ids 0..d-1 read one normed feature each
    rows[d + 3] = 1.0             # id d+3 sums the normed features
    x = f32_round(rng.standard_normal((5, d)) * 3.0)
    got = M.lm_logits(cfg, _LmRows(rows), x, chunk=7)   # chunks that do not divide V
    hn = _rms_bf16(x)
    assert got.dtype == np.float32 and got.shape == (5, V)
    assert np.array_equal(got[:, :d], hn.astype(np.float32))
    assert np.array_equal(got[:, d + 3], hn.sum(axis=1).astype(np.float32))
    assert np.all(got[:, d:d + 3] == 0) and np.all(got[:, d + 4:] == 0)
    # chunking over the vocabulary does not change a logit
    W2 = _LmRows(bf16_round(rng.standard_normal((V, d))))
    assert np.array_equal(M.lm_logits(cfg, W2, x, chunk=V), M.lm_logits(cfg, W2, x, chunk=3))
    # the final RMSNorm is applied: with eps 0 a power-of-two scale of the
    # stream is exact through the norm and changes no logit
    cfg0 = M.ModelConfig(n_layers=1, d_model=d, n_q_heads=4, n_kv_heads=4, head_dim=4, n_experts=4, top_k=2,
                         d_ff=8, vocab=V, rms_eps=0.0)
    assert np.array_equal(M.lm_logits(cfg0, W2, x * 4.0, chunk=V), M.lm_logits(cfg0, W2, x, chunk=V))


# ---- the layer's halves, as the stage checks call them ----------------------------

def test_layer_halves_compose_to_the_layer_and_pin_the_attention_half():
    # attention_block returns the closed-form stream after the uniform
    # attention residual; moe_block on it reproduces the whole layer; the
    # router alone makes moe_block's routing decisions
    rng = np.random.default_rng(23)
    d, Hq, Hkv, hd, E, k, f = 16, 4, 2, 4, 6, 2, 8
    G = Hq // Hkv
    cfg = _cfg(d, Hq, Hkv, hd, E, k, f)
    lw = _wired_layer(rng, d, Hq, Hkv, hd, E, f, zero_down=False)
    n = 6
    x = f32_round(rng.standard_normal((1, n, d)))
    kk = np.zeros((1, n, Hkv, hd), np.float32)
    vv = np.zeros((1, n, Hkv, hd), np.float32)
    xm = M.attention_block(cfg, lw, x, kk, vv, 0, causal=False, append=False)
    mean = _rms_bf16(x[0])[:, :Hkv * hd].mean(axis=0)
    want = np.concatenate([mean[(h // G) * hd:(h // G + 1) * hd] for h in range(Hq)])
    assert np.array_equal(xm[0], f32_round(x[0] + bf16_round(np.broadcast_to(want, (n, d)))))
    y, rec = M.moe_block(cfg, lw, xm)
    y2, rec2 = M.layer_forward(cfg, lw, x, kk, vv, 0, causal=False, append=False)
    assert np.array_equal(y, y2)
    r = M.router_block(cfg, lw, xm)
    for a, b in zip(r, rec):
        assert np.array_equal(np.asarray(a), np.asarray(b))
    # the router's choice is the top-k of its logits
    logits = np.asarray(r[3]).reshape(n, E)
    for t in range(n):
        assert list(np.asarray(r[0]).reshape(n, k)[t]) == list(np.argsort(-logits[t], kind="stable")[:k])


def test_router_weights_alone_equal_the_layer_router():
    cfg = M.ModelConfig(n_layers=2, d_model=64, n_q_heads=2, n_kv_heads=1, head_dim=32, n_experts=8, top_k=2,
                        d_ff=64, vocab=256)
    W = M.Weights(cfg, seed=3)
    wr1 = W.router(1)["wr"]
    assert np.array_equal(wr1, W.layer(1)["wr"])
    assert not np.array_equal(W.router(0)["wr"], wr1)


def test_forced_routing_uses_the_named_experts_with_their_own_softmax_weights():
    # forcing the router's own choice changes nothing; forcing other experts
    # takes exactly those, weighted by the softmax of their own logits
    rng = np.random.default_rng(24)
    d, Hq, Hkv, hd, E, k, f = 16, 4, 2, 4, 6, 2, 8
    cfg = _cfg(d, Hq, Hkv, hd, E, k, f)
    lw = _wired_layer(rng, d, Hq, Hkv, hd, E, f, zero_down=False)
    n = 5
    xm = f32_round(rng.standard_normal((1, n, d)))
    y, (idx, w, margin, rlog) = M.moe_block(cfg, lw, xm)
    y2, (idx2, w2, _, _) = M.moe_block(cfg, lw, xm, force_idx=idx)
    assert np.array_equal(y, y2) and np.array_equal(idx, idx2) and np.array_equal(w, w2)
    other = (np.asarray(idx) + 1) % E
    y3, (idx3, w3, margin3, rlog3) = M.moe_block(cfg, lw, xm, force_idx=other)
    assert np.array_equal(idx3, other) and np.array_equal(margin3, margin) and np.array_equal(rlog3, rlog)
    lg = np.asarray(rlog).reshape(n, E)
    for t in range(n):
        sel = lg[t, np.asarray(other).reshape(n, k)[t]]
        e = np.exp(sel - sel.max())
        assert np.array_equal(np.asarray(w3).reshape(n, k)[t], f32_round(e / e.sum()))
    assert not np.array_equal(y3, y)
    # layer_forward returns the router's own choice when forced
    kk = np.zeros((1, n, Hkv, hd), np.float32)
    vv = np.zeros((1, n, Hkv, hd), np.float32)
    x = f32_round(rng.standard_normal((1, n, d)))
    _, (own, _, _, _) = M.layer_forward(cfg, lw, x, kk, vv, 0, causal=False, append=False)
    _, (own2, _, _, _) = M.layer_forward(cfg, lw, x, kk, vv, 0, causal=False, append=False,
                                         force_idx=(np.asarray(own) + 1) % E)
    assert np.array_equal(own, own2)
