"""The plain C++ oracle (oracle/dg_oracle.cpp): its generator and bf16
rounding against fixed values, then whole rounds against the numpy oracle on
the same seeded weights and inputs.  The two implementations share no code
(only the seeded weight generator): the numpy oracle is pinned by its own
tests, and a second implementation that agrees with it at every decision
point rules out mistakes that only one of them could make."""

import os

import numpy as np
import pytest

import oracle
import synth
from oracle import cpp
from oracle import decode as OD
from oracle import sampler as OS
from oracle.numerics import bf16_round

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")
TINY = dict(n_layers=2, d_model=256, n_q_heads=8, n_kv_heads=8, head_dim=32, n_experts=16, top_k=2,
            d_ff=512, vocab=4096)


def _kat():
    """(counter and key words, output words) per line: ctr0-3 key0-1 out0-3 in hex."""
    rows = []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            w = [int(x, 16) for x in line.split()]
            rows.append((w[:6], w[6:10]))
    return rows


def test_philox_reproduces_the_published_known_answers():
    out = np.zeros(4, np.uint32)
    rows = _kat()
    assert rows
    for ins, want in rows:
        cpp.lib().dgo_philox(*ins, out.ctypes.data)
        assert [int(x) for x in out] == want


def test_bf16_rounding_agrees_with_the_numpy_oracles_bit_formulation():
    """Two formulations of round-to-nearest-even to 8 significant bits: the
    C++ side scales to the integer grid and rounds, the numpy side masks the
    double's mantissa; ties, near-ties, subnormal flushes and signs."""
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-40, 40, 20000),
                        [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 2 ** -126, 2 ** -127,
                         -(2 ** -130), 255.5, 3.0 * 2 ** 100]])
    near = (1.0 + np.arange(1, 128) * 2 ** -7 + 2 ** -8)  # exact halfway points between bf16 neighbours
    x = np.concatenate([x, near, np.nextafter(near, 0), np.nextafter(near, 4)])
    got = np.array([cpp.lib().dgo_bf16(float(v)) for v in x])
    want = bf16_round(x)
    assert np.array_equal(got.view(np.uint64), want.view(np.uint64))


def _state_for_cpp(state, d):
    B, N = state.tokens.shape
    return {"tokens": state.tokens.copy(), "sc": np.ascontiguousarray(state.sc, dtype=np.float64).copy(),
            "prev_argmax": state.prev_argmax.copy(), "done": state.done.astype(np.uint8),
            "locked": (state.locked if state.locked is not None else np.zeros((B, N), bool)).astype(np.uint8)}


def _run(cfg, samp, rounds, batch, ctx=64):
    """Both oracles from the same seeded weights: the context encoded
    causally by each, then `rounds` rounds, the C++ side starting each round
    from the numpy oracle's state (a decision taken differently at a near-tie
    does not carry over).  Returns what was compared."""
    ocfg = oracle.ModelConfig(**cfg)
    W = oracle.Weights(ocfg, seed=0)
    m = cpp.Model(ocfg, seed=0)
    kv = oracle.KVCache(ocfg, batch, ctx + 256)
    cache = cpp.Cache(ocfg, batch, ctx + 256)
    toks = synth.context_tokens(batch, ctx, 1234, ocfg.vocab).astype(np.int64)
    OD.encode_context(ocfg, W, kv, toks)
    cpp.encode_context(m, cache, toks)
    assert cache.length == kv.length == ctx
    for l in range(ocfg.n_layers):
        assert np.array_equal(cache.k[l][:, :ctx], kv.k[l][:, :ctx]) and np.array_equal(cache.v[l][:, :ctx],
                                                                                        kv.v[l][:, :ctx])
    sc = OS.SamplerConfig(**samp)
    cs = cpp.sampler(**samp)
    canvas = OD.init_canvas(sc.seed, 0, batch, 256, ocfg.vocab)
    assert np.array_equal(canvas, cpp.init_canvas(sc.seed, 0, batch, 256, ocfg.vocab))
    state = OD.new_state(canvas, ocfg.d_model)
    report = {"decisions": 0, "excused": 0, "logit_rel": 0.0, "locked": 0, "stopped": 0, "kept": 0}
    for s in range(rounds):
        cst = _state_for_cpp(state, ocfg.d_model)
        before = state.tokens.copy()
        committed = None if state.locked is None else state.locked.copy()
        want = OD.denoise_step(ocfg, W, kv, state, sc, 0, s, keep_logits=True, record_routing=True)
        got = cpp.denoise_step(m, cache, cst, cs, 0, s)
        # logits: fp32 values from double accumulations in another order
        rel = np.abs(got["logits"] - want.logits).max() / np.abs(want.logits).max()
        report["logit_rel"] = max(report["logit_rel"], float(rel))
        assert rel <= 1e-6, (s, rel)
        # routing: the same experts wherever the router's own ranking is not a near-tie
        for l, (idx, _w, margin, _x, _rl) in enumerate(want.routing):
            ok = margin > 1e-9
            assert np.array_equal(got["route_idx"][l][ok], idx[ok]), (s, l)
            report["decisions"] += int(ok.sum())
            report["excused"] += int((~ok).sum())
        np.testing.assert_allclose(got["entropy"], want.entropy, rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(got["pmax"], want.pmax, rtol=1e-9, atol=1e-15)
        np.testing.assert_allclose(got["mean_entropy"], want.mean_entropy, rtol=1e-9)
        a_ok, s_ok = want.argmax_margin > 1e-6, want.sample_margin > 1e-5
        assert np.array_equal(got["argmax"][a_ok], want.argmax[a_ok]), s
        assert np.array_equal(got["sample"][s_ok], want.sample[s_ok]), s
        report["decisions"] += int(a_ok.sum() + s_ok.sum())
        report["excused"] += int((~a_ok).sum() + (~s_ok).sum())
        if a_ok.all() and s_ok.all():
            assert np.array_equal(got["lock"].astype(bool), want.lock), s
            assert np.array_equal(got["stop"].astype(bool), want.stop) and np.array_equal(
                got["final"].astype(bool), want.final), s
            assert np.array_equal(cst["tokens"], state.tokens), s
            assert np.array_equal(cst["done"].astype(bool), state.done), s
            if ocfg.self_cond:
                assert np.array_equal(cst["sc"], state.sc), s
        report["locked"] += int(want.lock.sum())
        report["stopped"] += int(want.stop.sum())
        if committed is not None and samp.get("persistent_lock"):
            report["kept"] += int((committed & (state.tokens == before)).sum())
    print(report)
    return report


def test_the_tiny_models_4_round_loop_agrees():
    """The tiny configuration's loop: context 64, one canvas, 4 rounds,
    lock above 0.9, Philox seed 1234."""
    rep = _run(TINY, dict(max_steps=4, lock_threshold=0.9, seed=1234), rounds=4, batch=1)
    # per round: each layer's routing of 256 tokens, then 256 argmax and 256 samples
    assert rep["decisions"] + rep["excused"] == 4 * (2 * 256 + 2 * 256)
    assert rep["excused"] <= 0.01 * rep["decisions"], rep


def test_self_conditioning_entropy_budget_and_two_canvases_agree():
    """Self-conditioning input (the expected embedding), the entropy-budget
    lock rule with room for a few positions, two canvases."""
    rep = _run(dict(TINY, self_cond=True), dict(max_steps=6, lock_policy=OS.LOCK_ENTROPY_CUMSUM,
                                                lock_threshold=25.0, seed=77), rounds=2, batch=2)
    assert rep["decisions"] > 0


def test_the_stop_freezes_both_canvases_and_the_next_round_leaves_them():
    """A stop threshold every round reaches: round 0 turns each canvas into
    its argmax and freezes it; round 1 changes nothing."""
    rep = _run(TINY, dict(max_steps=8, stop_entropy=100.0, seed=5), rounds=2, batch=2)
    assert rep["stopped"] == 2, rep


def test_topk_self_conditioning_and_the_persistent_lock_agree():
    """The top-k (16) self-conditioning input and the persistent lock, with a
    threshold near the median largest probability: about half the positions
    lock in a round and keep their tokens in the rounds after."""
    rep = _run(dict(TINY, self_cond=True), dict(max_steps=8, seed=5, selfcond_topk=16, persistent_lock=True,
                                                lock_threshold=7.6e-4), rounds=3, batch=1)
    assert rep["locked"] > 0 and rep["kept"] > 0, rep


def test_grouped_query_attention_and_wider_routing_agree():
    """Two query heads per kv head (head_dim 64), top-4 of 32 experts, three
    layers, a longer context and a round later in the block."""
    cfg = dict(n_layers=3, d_model=512, n_q_heads=8, n_kv_heads=4, head_dim=64, n_experts=32, top_k=4,
               d_ff=256, vocab=2048)
    rep = _run(cfg, dict(max_steps=12, lock_threshold=1e-3, seed=99), rounds=2, batch=1, ctx=200)
    assert rep["decisions"] + rep["excused"] == 2 * (3 * 256 + 2 * 256)
    assert rep["excused"] <= 0.01 * rep["decisions"], rep


def test_round_invariants_of_the_cpp_oracle():
    """What the pages fix, checked on the C++ oracle's own outputs: entropy in
    [0, ln V] and 1/V <= pmax <= 1; a locked position's next token is its
    sample; the stop fires exactly when the mean entropy is below the
    threshold (thresholds just above and just below the round's value)."""
    ocfg = oracle.ModelConfig(**TINY)
    m = cpp.Model(ocfg, seed=0)
    V = ocfg.vocab

    def one_round(stop_entropy, lock_threshold):
        cache = cpp.Cache(ocfg, 1, 64 + 256)
        cpp.encode_context(m, cache, synth.context_tokens(1, 64, 1234, V).astype(np.int64))
        st = {"tokens": cpp.init_canvas(3, 0, 1, 256, V), "sc": np.zeros((1, 256, ocfg.d_model)),
              "prev_argmax": np.full((1, 256), -1, np.int64), "done": np.zeros(1, np.uint8),
              "locked": np.zeros((1, 256), np.uint8)}
        o = cpp.denoise_step(m, cache, st, cpp.sampler(max_steps=48, seed=3, stop_entropy=stop_entropy,
                                                       lock_threshold=lock_threshold), 0, 0)
        return o, st

    o, st = one_round(0.5, 7.6e-4)
    assert np.all(o["entropy"] >= 0) and np.all(o["entropy"] <= np.log(V) + 1e-12)
    assert np.all(o["pmax"] >= 1.0 / V - 1e-15) and np.all(o["pmax"] <= 1.0)
    lock = o["lock"].astype(bool)
    assert 0 < lock.sum() < lock.size
    assert np.array_equal(st["tokens"][lock], o["sample"][lock])
    mh = float(o["mean_entropy"][0])
    below, _ = one_round(np.nextafter(mh, np.inf), 7.6e-4)
    above, _ = one_round(mh, 7.6e-4)
    assert below["stop"][0] == 1 and below["final"][0] == 1
    assert above["stop"][0] == 0 and above["final"][0] == 0
