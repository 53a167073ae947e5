"""Pins of the oracle's vocabulary statistics, sampler, lock rules, stop rule,
temperature schedule and expected embedding (no GPU)."""

import itertools
import math

import numpy as np
import pytest

from oracle import sampler as S
from oracle import philox


def test_uniform_logits_entropy_is_log_v():
    for V in (4096, 262144):
        H, pmax, amax, p = S.position_stats(np.zeros(V, np.float32))
        assert abs(H - math.log(V)) < 1e-9
        assert abs(pmax - 1.0 / V) < 1e-15
        assert amax == 0  # ties go to the lower id
        assert abs(p.sum() - 1.0) < 1e-12
    assert abs(math.log(262144) - 12.4766) < 1e-4


def test_two_level_logits_closed_form():
    # one logit a, V-1 logits 0: p1 = e^a / (e^a + V - 1)
    V, a = 1000, 3.0
    l = np.zeros(V, np.float32)
    l[17] = a
    H, pmax, amax, p = S.position_stats(l)
    Z = math.exp(a) + V - 1
    p1, p0 = math.exp(a) / Z, 1.0 / Z
    assert abs(pmax - p1) < 1e-12 and amax == 17
    assert abs(H - (-(p1 * math.log(p1)) - (V - 1) * p0 * math.log(p0))) < 1e-10


def test_entropy_bounds_random_logits():
    rng = np.random.default_rng(0)
    for scale in (0.01, 1.0, 30.0):
        l = (rng.standard_normal(5000) * scale).astype(np.float32)
        H, pmax, amax, p = S.position_stats(l)
        assert 0.0 <= H <= math.log(5000) + 1e-12
        assert abs(p.sum() - 1.0) < 1e-12
        assert amax == int(np.argmax(l))


def test_gumbel_max_frequencies_match_softmax():
    logits = np.array([0.0, 0.5, 1.0, -1.0, 2.0, 0.2, -0.3, 1.5], np.float32)
    inv_t = np.float32(1.0 / 0.7)
    n = 60000
    # independent draws: 60000 positions of the counter space, two Philox
    # blocks (c0 = 0, 1) give the 8 per-id words of each draw
    pos = np.arange(n, dtype=np.uint64)
    words = np.stack(philox.method_draw(99, philox.PURPOSE_GUMBEL, 0, 0, 0, pos, 0), axis=1)
    words = np.concatenate([words, np.stack(philox.method_draw(99, philox.PURPOSE_GUMBEL, 0, 0, 0,
                                                               pos, 1), axis=1)], axis=1)
    keys = (logits * inv_t)[None, :] + (-np.log(-np.log(philox.gumbel_u(words))))
    counts = np.bincount(np.argmax(keys, axis=1), minlength=8)
    p = np.exp(logits.astype(np.float64) * float(inv_t))
    p /= p.sum()
    exp = n * p
    chi2 = float(((counts - exp) ** 2 / exp).sum())
    assert chi2 < 40, chi2  # 7 degrees of freedom; p < 1e-5 beyond ~33


def test_gumbel_sample_low_temperature_is_argmax():
    rng = np.random.default_rng(1)
    l = rng.standard_normal(300).astype(np.float32)
    words = philox.gumbel_words(5, 0, 0, 0, 3, 300)
    tok, _ = S.gumbel_sample(l, np.float32(1e6), words)
    assert tok == int(np.argmax(l))


def test_gumbel_words_layout():
    w = philox.gumbel_words(11, 2, 1, 3, 7, 10)
    blk = philox.method_draw(11, philox.PURPOSE_GUMBEL, 2, 1, 3, 7, 2)  # c0 = 2 covers ids 8..11
    assert int(w[8]) == int(blk[0]) and int(w[9]) == int(blk[1])


def test_temperature_schedule():
    assert S.temperature(0, 48) == 0.8
    assert abs(S.temperature(47, 48) - 0.4) < 1e-15
    assert abs(S.temperature(1, 3) - 0.6) < 1e-15
    assert [round(S.temperature(s, 4), 4) for s in range(4)] == [0.8, 0.6667, 0.5333, 0.4]
    assert S.temperature(0, 1) == 0.8


def test_prob_lock_is_strict_threshold():
    pmax = np.array([0.9, 0.9 + 1e-9, 0.5, 0.99])
    assert list(S.lock_mask(np.zeros(4), pmax, S.LOCK_PROB, 0.9)) == [False, True, False, True]


def _cumsum_lock_brute(H, theta):
    """Independent formulation: i is locked iff the total entropy of all
    positions ordered at or before i (by (H, index)) is <= theta."""
    n = len(H)
    out = np.zeros(n, bool)
    for i in range(n):
        before = [j for j in range(n) if (H[j], j) <= (H[i], i)]
        out[i] = sum(H[j] for j in before) <= theta
    return out


def test_cumsum_lock_matches_enumeration():
    rng = np.random.default_rng(2)
    for trial in range(300):
        H = rng.choice([0.0, 0.01, 0.02, 0.05, 0.1, 0.3], size=8) * rng.uniform(0.5, 1.5)
        if trial % 3 == 0:
            H = rng.exponential(0.04, size=8)
        got = S.lock_mask(H, np.zeros(8), S.LOCK_ENTROPY_CUMSUM, 0.1)
        assert np.array_equal(got, _cumsum_lock_brute(list(H), 0.1)), H
    # every subset size reachable; the crossing position is not locked
    H = np.array([0.05, 0.04, 0.02, 0.5])
    assert list(S.lock_mask(H, None, S.LOCK_ENTROPY_CUMSUM, 0.1)) == [False, True, True, False]


def test_stop_fires_exactly_below_threshold():
    assert S.stop_flag(0.4999, 0.5, False, 0, None, None)
    assert not S.stop_flag(0.5, 0.5, False, 0, None, None)
    a = np.array([1, 2, 3])
    assert not S.stop_flag(0.0, 0.5, True, 0, a, None)          # never at step 0
    assert S.stop_flag(0.0, 0.5, True, 3, a, a.copy())
    assert not S.stop_flag(0.0, 0.5, True, 3, a, np.array([1, 2, 4]))


def test_stop_on_constructed_logits():
    # two-level logits with entropy straddling the threshold
    V = 100
    def H_of(a):
        l = np.zeros(V, np.float32)
        l[0] = a
        return S.position_stats(l)[0]
    lo, hi = H_of(12.0), H_of(2.0)
    assert lo < 0.5 < hi
    assert S.stop_flag(np.mean([lo] * 4), 0.5, False, 1, None, None)
    assert not S.stop_flag(np.mean([hi] * 4), 0.5, False, 1, None, None)
    mixed = np.mean([lo, lo, lo, hi])
    assert S.stop_flag(mixed, 0.5, False, 1, None, None) == (mixed < 0.5)


def test_expected_embedding_one_hot_returns_row():
    from oracle.model import ModelConfig, Weights
    cfg = ModelConfig(1, 16, 1, 1, 16, 1, 1, 16, 64)
    W = Weights(cfg, seed=3)
    p = np.zeros((2, 64))
    p[0, 5] = 1.0
    p[1, 63] = 1.0
    e = S.expected_embedding(p, W, chunk=16)
    assert np.array_equal(e[0], W.emb_chunk(5, 1)[0])
    assert np.array_equal(e[1], W.emb_chunk(63, 1)[0])
    # uniform p gives the mean row (within bf16 rounding of the result)
    e = S.expected_embedding(np.full((1, 64), 1 / 64), W, chunk=64)
    assert np.allclose(e[0], W.emb_chunk(0, 64).mean(0), atol=2 ** -9 * np.abs(e).max() + 1e-6)


def test_renoise_uniform_and_deterministic():
    a = S.renoise_tokens(1, 0, 2, 3, 256, 4096)
    b = S.renoise_tokens(1, 0, 2, 3, 256, 4096)
    c = S.renoise_tokens(1, 0, 2, 4, 256, 4096)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    assert a.min() >= 0 and a.max() < 4096


def test_selfcond_probs_round_only_the_stored_logits():
    from oracle.numerics import bf16_round
    # logits that bf16 holds exactly: the plain softmax
    l = np.array([1.0, 0.5, -2.0, 0.25, 0.0], np.float32)
    p = S.selfcond_probs(l)
    e = np.exp(l.astype(np.float64) - 1.0)
    assert np.allclose(p, e / e.sum(), rtol=0, atol=1e-15)
    # a logit bf16 cannot hold: its numerator uses the rounded value, the
    # normaliser (max and sum) the exact fp32 logits
    a = np.float32(1.0 + 2.0 ** -10)          # between two bf16 values (1 and 1 + 2^-7)
    l = np.array([a, 0.0, 0.0], np.float32)
    p = S.selfcond_probs(l)
    Z = 1.0 + 2.0 * np.exp(-float(a))
    assert float(bf16_round(a)) == 1.0
    assert p[0] == np.exp(1.0 - float(a)) / Z
    assert p[1] == p[2] == np.exp(-float(a)) / Z
    assert abs(p.sum() - 1.0) > 1e-6   # no longer a distribution: the rounding is visible


class _EmbRows:
    """Stands in for the weights: embedding rows of a given matrix."""

    def __init__(self, rows):
        self.rows = rows

        class _C:
            d_model = rows.shape[1]
        self.cfg = _C()

    def emb_rows(self, toks):
        return self.rows[np.asarray(toks)]


def test_expected_embedding_topk_selection_and_weights():
    from oracle.numerics import bf16_round
    rng = np.random.default_rng(11)
    V, d = 40, 8
    E = bf16_round(rng.standard_normal((V, d)))
    W = _EmbRows(E)
    # k = 1: the embedding row of the largest bf16 logit
    l = rng.standard_normal((3, V)).astype(np.float32)
    e, ids = S.expected_embedding_topk(l, W, 1)
    for t in range(3):
        am = int(np.argmax(bf16_round(l[t].astype(np.float64))))
        assert ids[t, 0] == am and np.array_equal(e[t], bf16_round(E[am]))
    # ties go to the lower ids: equal logits select ids 0..k-1 with equal weights
    l = np.zeros((1, V), np.float32)
    e, ids = S.expected_embedding_topk(l, W, 4)
    assert list(ids[0]) == [0, 1, 2, 3]
    assert np.array_equal(e[0], bf16_round(bf16_round(np.full(4, 0.25)) @ E[:4]))
    # brute force: the selected set is the k largest bf16 logits, the weights their softmax
    l = rng.standard_normal((2, V)).astype(np.float32) * 3
    k = 7
    e, ids = S.expected_embedding_topk(l, W, k)
    for t in range(2):
        lb = bf16_round(l[t].astype(np.float64))
        ranked = sorted(range(V), key=lambda v: (-lb[v], v))[:k]
        assert list(ids[t]) == sorted(ranked)
        w = np.exp(lb[sorted(ranked)] - lb[ranked[0]])
        want = bf16_round(bf16_round(w / w.sum()) @ E[sorted(ranked)])
        assert np.array_equal(e[t], want)
    # k >= V keeps every id
    e, ids = S.expected_embedding_topk(l, W, V + 5)
    assert ids.shape == (2, V)
