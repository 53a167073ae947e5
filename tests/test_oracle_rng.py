"""Pins of the oracle's random draws and of the seeded input generator.

Philox4x32-10 is pinned to its published known-answer vectors and to a
second, independent implementation (the C generator in synth/).  The draws
built on it are pinned by their distributions (chi-square)."""

import os

import numpy as np
import pytest

import synth
from oracle import philox
from oracle.numerics import bf16_bits_to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _kat():
    rows = []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            w = [int(x, 16) for x in line.split()]
            rows.append((w[:4], w[4:6], w[6:10]))
    return rows


@pytest.mark.parametrize("ctr,key,out", _kat())
def test_philox_known_answers_oracle(ctr, key, out):
    got = philox.philox4x32_10(*ctr, *key)
    assert [int(v) for v in got] == out


@pytest.mark.parametrize("ctr,key,out", _kat())
def test_philox_known_answers_synth(ctr, key, out):
    assert list(synth.philox4x32_10(ctr, key)) == out


def test_philox_two_implementations_agree():
    rng = np.random.default_rng(7)
    for _ in range(200):
        ctr = [int(v) for v in rng.integers(0, 2**32, 4)]
        key = [int(v) for v in rng.integers(0, 2**32, 2)]
        a = [int(v) for v in philox.philox4x32_10(*ctr, *key)]
        assert a == list(synth.philox4x32_10(ctr, key))


def test_philox_vectorised_matches_scalar():
    c0 = np.arange(1000, dtype=np.uint64)
    w = philox.philox4x32_10(c0, 3, 5, 7, 11, 13)
    for i in (0, 1, 517, 999):
        s = synth.philox4x32_10([i, 3, 5, 7], [11, 13])
        assert tuple(int(x[i]) for x in w) == s


def test_uniform_token_chi_square():
    V = 64
    w0, _, _, _ = philox.method_draw(1234, philox.PURPOSE_RENOISE, 0, 0, 0,
                                     np.arange(64000, dtype=np.uint64))
    toks = philox.uniform_token(w0, V)
    assert toks.min() >= 0 and toks.max() < V
    counts = np.bincount(toks, minlength=V)
    exp = toks.size / V
    chi2 = float(((counts - exp) ** 2 / exp).sum())
    # 63 degrees of freedom: mean 63, sd ~11.2; 120 is beyond p = 1e-5
    assert chi2 < 120, chi2


def test_uniform_token_exact_edges():
    # floor(r * V / 2^32): r = 0 -> 0, r = 2^32 - 1 -> V - 1
    assert int(philox.uniform_token(0, 262144)) == 0
    assert int(philox.uniform_token(2**32 - 1, 262144)) == 262143
    assert int(philox.uniform_token(2**31, 4096)) == 2048


def test_gumbel_u_range_and_exactness():
    u = philox.gumbel_u(np.array([0, 2**32 - 1, 511, 512], dtype=np.uint64))
    assert u.dtype == np.float32
    assert u[0] == np.float32(0.5 * 2.0 ** -23)
    assert u[1] == np.float32(1.0 - 0.5 * 2.0 ** -23)
    assert u[2] == u[0] and u[3] == np.float32(1.5 * 2.0 ** -23)
    assert np.all((u > 0) & (u < 1))


def test_synth_weights_moments_and_bounds():
    w = bf16_bits_to_f64(synth.bf16_tensor((512, 1024), 0, synth.layer_tid(0, synth.KIND_WQ)))
    assert abs(w.mean()) < 2e-4
    assert abs(w.std() - 0.02) < 2e-4
    # a sum of four uniforms is bounded by 2 * sqrt(3) standard deviations
    assert np.abs(w).max() <= 0.02 * 2 * np.sqrt(3) * 1.004


def test_synth_rows_window_matches_whole():
    tid = synth.layer_tid(3, synth.KIND_WG)
    whole = synth.bf16_tensor((40, 96), 5, tid)
    part = synth.bf16_rows(17, 9, 96, 5, tid)
    assert np.array_equal(whole[17:26], part)


def test_synth_tokens_uniform():
    toks = synth.tokens(40000, 9, synth.ctx_tid(0), 50)
    counts = np.bincount(toks, minlength=50)
    exp = toks.size / 50
    assert float(((counts - exp) ** 2 / exp).sum()) < 100
