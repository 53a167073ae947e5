"""The work schedules of the grouped (mixture-of-experts) products, enumerated
on the host through the C ABI (no GPU): every (expert, 128-row weight tile,
chunk of at most bn tokens) is one job of exactly one CTA, with the right
rows, columns and k range; on CTA pairs the two ranks of a unit share the
chunk and take consecutive tiles, the only empty tile being the missing
second tile of an odd tile count; units run expert, then tile, then chunk."""

import ctypes
import os

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "discrete_diffusion_moe_b200", "libdg.so")
I32 = ctypes.c_int32
P = ctypes.c_void_p


@pytest.fixture(scope="module")
def fn():
    lib = ctypes.CDLL(LIB)
    f = lib.dg_test_grouped_schedule
    f.restype = I32
    f.argtypes = [I32, I32, I32, P, I32, I32, P, I32, P]
    return f


def _jobs(fn, pair, R, sizes, K, bn):
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    n = I32(0)
    st = fn(pair, R, len(sizes), off.ctypes.data, K, bn, None, 0, ctypes.byref(n))
    assert st == 0
    jobs = np.zeros((max(n.value, 1), 10), np.int32)
    st = fn(pair, R, len(sizes), off.ctypes.data, K, bn, jobs.ctypes.data, n.value, ctypes.byref(n))
    assert st == 0
    return off, jobs[:n.value]


def _check(fn, pair, R, sizes, K, bn):
    off, jobs = _jobs(fn, pair, R, sizes, K, bn)
    m_tiles = (R + 127) // 128
    want = {(g, t, c) for g, rows in enumerate(sizes) for t in range(m_tiles) for c in range(-(-rows // bn))}
    seen = []
    for u, r, g, t, a0, mv, n0, nv, kb, bmap in jobs:
        rows = sizes[g]
        c = (n0 - off[g]) // bn
        assert n0 == off[g] + c * bn and 0 <= c < -(-rows // bn)
        assert nv == min(bn, rows - c * bn) and nv >= 1
        assert kb == K // 64
        assert a0 == g * R + t * 128
        if mv <= 0:  # the missing second tile of an odd tile count, pairs only
            assert pair and r == 1 and t == m_tiles and m_tiles % 2 == 1
            continue
        assert mv == min(128, R - t * 128)
        seen.append((g, t, c))
        if pair:
            half = ((nv + 15) & ~15) // 2
            box = [8, min(32, bn // 2), bn // 2]
            assert half <= box[bmap] and (bmap == 0 or half > box[bmap - 1])
        else:
            assert bmap == -1
    assert len(seen) == len(set(seen)) and set(seen) == want
    ranks = 2 if pair else 1
    assert len(jobs) % ranks == 0
    units = jobs.reshape(-1, ranks, 10)
    assert np.array_equal(units[:, 0, 0], np.arange(len(units)))
    if pair:  # both ranks of a unit: one chunk, consecutive tiles
        assert np.array_equal(units[:, 0, 6], units[:, 1, 6]) and np.array_equal(units[:, 0, 2], units[:, 1, 2])
        assert np.all(units[:, 1, 3] == units[:, 0, 3] + 1) and np.all(units[:, 0, 3] % 2 == 0)
    # unit order: expert, then tile (pair), then chunk
    key = [(j[2], j[3] // ranks, j[6]) for j in units[:, 0]]
    assert key == sorted(key)


@pytest.mark.parametrize("pair", [1, 0])
@pytest.mark.parametrize("R,K", [(128, 64), (200, 192), (384, 128), (1408, 2816), (2816, 704)])
@pytest.mark.parametrize("bn", [16, 32, 64, 128])
def test_every_tile_and_chunk_is_one_job(fn, pair, R, K, bn):
    rng = np.random.default_rng(R + K + bn + pair)
    sizes = [int(x) for x in rng.integers(0, 3 * bn, size=9)]
    sizes[2] = 0
    sizes[5] = bn  # exactly one full chunk
    _check(fn, pair, R, sizes, K, bn)


def test_single_cta_schedule_at_256_token_chunks(fn):
    _check(fn, 0, 1408, [300, 0, 256, 1, 513], 2816, 256)


def test_deep_layer_routing(fn):
    # a deep layer of the full-size step: ~12 experts with ~170 tokens each
    sizes = [0] * 128
    for e, n in zip(range(3, 128, 10), [170, 171, 169, 172, 168, 170, 170, 171, 169, 170, 170, 170, 40]):
        sizes[e] = n
    _check(fn, 1, 1408, sizes, 2816, 128)
    _check(fn, 1, 2816, sizes, 704, 128)


def test_rejects_bad_arguments(fn):
    off = np.array([0, 5, 3], np.int32)  # decreasing
    n = I32(0)
    assert fn(1, 128, 2, off.ctypes.data, 64, 32, None, 0, ctypes.byref(n)) != 0
    good = np.array([0, 5, 9], np.int32)
    assert fn(1, 128, 2, good.ctypes.data, 64, 256, None, 0, ctypes.byref(n)) != 0  # pairs: bn <= 128
    assert fn(0, 128, 2, good.ctypes.data, 96, 32, None, 0, ctypes.byref(n)) != 0   # K % 64
    assert fn(0, 128, 2, good.ctypes.data, 64, 48, None, 0, ctypes.byref(n)) != 0   # bn not a power of 2
    assert fn(0, 128, 2, good.ctypes.data, 64, 32, None, 0, ctypes.byref(n)) == 0 and n.value > 0
