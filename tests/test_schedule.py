"""The work schedules of the GEMM core, enumerated on the host through the C
ABI (no GPU).  Grouped (mixture-of-experts) products: every (expert, 128-row
weight tile, chunk of at most bn tokens) is one job of exactly one CTA, with
the right rows, columns and k range; on CTA pairs the two ranks of a unit
share the chunk and take consecutive tiles, the only empty tile being the
missing second tile of an odd tile count; units run expert, then tile, then
chunk.  Dense products: every (A tile, column tile) is covered once per k
split, the splits partition the k blocks, and units walk the splits, then
the column tiles (or the A tiles).  The one-launch expert block: the chunk
counters its down units wait on, and the unit order that makes those waits
end."""

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


# ---- dense products (projections, LM head, expected embedding) ------------------

@pytest.fixture(scope="module")
def dense_fn():
    lib = ctypes.CDLL(LIB)
    f = lib.dg_test_dense_schedule
    f.restype = I32
    f.argtypes = [I32, I32, I32, I32, I32, I32, I32, P, I32, P]
    return f


def _dense_jobs(fn, M, N, K, bn, ks, mt, n_fast):
    n = I32(0)
    assert fn(M, N, K, bn, ks, mt, n_fast, None, 0, ctypes.byref(n)) == 0
    jobs = np.zeros((max(n.value, 1), 8), np.int32)
    assert fn(M, N, K, bn, ks, mt, n_fast, jobs.ctypes.data, n.value, ctypes.byref(n)) == 0
    return jobs[:n.value]


@pytest.mark.parametrize("M,N,K,bn,ks,mt,n_fast", [
    (128, 16, 64, 16, 1, 1, 1), (5632, 256, 2816, 128, 3, 1, 1), (2816, 256, 2048, 64, 2, 2, 1),
    (384, 200, 320, 64, 5, 2, 0), (200, 1000, 704, 256, 1, 2, 1), (128 * 44 + 3, 33, 192, 32, 3, 2, 0),
    (256, 262144, 2816, 256, 1, 1, 0), (2816, 256, 262144 // 64 * 64, 128, 8, 1, 1)])
def test_dense_schedule_covers_every_tile_once(dense_fn, M, N, K, bn, ks, mt, n_fast):
    jobs = _dense_jobs(dense_fn, M, N, K, bn, ks, mt, n_fast)
    m_tiles, n_tiles, kbt = -(-M // 128), -(-N // bn), K // 64
    assert len(jobs) == -(-m_tiles // mt) * n_tiles * ks
    pieces = {}
    for u, t0, mte, mv, n0, nv, kb0, kb1 in jobs:
        assert t0 % mt == 0 and mte == min(mt, m_tiles - t0) and mte >= 1
        assert mv == min(128, M - 128 * t0) and mv >= 1
        assert n0 % bn == 0 and nv == min(bn, N - n0) and nv >= 1
        assert 0 <= kb0 < kb1 <= kbt
        for t in range(t0, t0 + mte):
            pieces.setdefault((t, n0 // bn), []).append((kb0, kb1))
    assert set(pieces) == {(t, c) for t in range(m_tiles) for c in range(n_tiles)}
    for key, ranges in pieces.items():  # the k splits partition the k blocks
        ranges.sort()
        assert len(ranges) == ks and ranges[0][0] == 0 and ranges[-1][1] == kbt, key
        assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:])), key
    # consecutive units: the k splits of one tile, then (n_fast) the column tiles of one A tile
    first = jobs[::ks]
    assert all(np.all(jobs[i * ks:(i + 1) * ks, 1] == first[i, 1]) and
               np.all(jobs[i * ks:(i + 1) * ks, 4] == first[i, 4]) for i in range(len(first)))
    if n_fast and n_tiles > 1:
        assert first[0, 1] == first[1, 1] and first[1, 4] == first[0, 4] + bn
    elif not n_fast and -(-m_tiles // mt) > 1:
        assert first[0, 4] == first[1, 4] and first[1, 1] == first[0, 1] + mt


def test_dense_schedule_rejects_bad_arguments(dense_fn):
    n = I32(0)
    assert dense_fn(128, 16, 64, 16, 2, 1, 1, None, 0, ctypes.byref(n)) != 0   # more splits than k blocks
    assert dense_fn(128, 16, 64, 16, 1, 3, 1, None, 0, ctypes.byref(n)) != 0   # mt 3
    assert dense_fn(128, 16, 100, 16, 1, 1, 1, None, 0, ctypes.byref(n)) != 0  # K % 64


@pytest.mark.parametrize("seed,E,k,T", [(0, 128, 8, 256), (1, 128, 8, 256), (2, 16, 2, 256), (3, 128, 8, 512)])
def test_fused_expert_block_dependencies(fn, seed, E, k, T):
    """The one-launch expert block (gate/up units, then down units, on CTA
    pairs; pair c takes units c, c + clusters, ...): a down unit of token chunk
    q waits until every CTA of the gate/up units of q has published, i.e. for
    2 x (gate/up tile pairs) arrivals.  On random routings: each chunk has
    exactly that many gate/up CTAs and one down unit per down tile pair, both
    phases number the chunks alike and within the counter array, and every
    pair reaches all of its gate/up units before its first down unit."""
    d, f, bn, clusters = 2816, 704, 128, 148
    rng = np.random.default_rng(seed)
    counts = np.bincount(np.concatenate([rng.choice(E, k, replace=False) for _ in range(T)]), minlength=E)
    sizes = [int(x) for x in counts]
    chunk_off = np.concatenate([[0], np.cumsum([-(-s // bn) for s in sizes])])
    n_chunks = int(chunk_off[-1])

    def units(R, K):
        off, jobs = _jobs(fn, 1, R, sizes, K, bn)
        out = {}
        for u, r, g, t, a0, mv, n0, nv, kb, bmap in jobs:
            out.setdefault(int(u), []).append(int(chunk_off[g] + (n0 - off[g]) // bn))
        assert all(len(set(v)) == 1 and len(v) == 2 for v in out.values())  # both ranks, one chunk
        return {u: v[0] for u, v in out.items()}

    up, down = units(2 * f, d), units(d, f)
    p_up, p_down = (2 * f // 128 + 1) // 2, (d // 128 + 1) // 2
    assert len(up) == p_up * n_chunks and len(down) == p_down * n_chunks
    arrivals = np.bincount([q for q in up.values()], minlength=n_chunks) * 2  # both CTAs of a unit add one
    assert np.all(arrivals == 2 * p_up)
    assert np.all(np.bincount([q for q in down.values()], minlength=n_chunks) == p_down)
    assert n_chunks <= T * k // 16 + E + 1  # the counters the workspace holds
    U1 = len(up)
    for c in range(clusters):
        mine = list(range(c, U1 + len(down), clusters))
        first_down = next((i for i, u in enumerate(mine) if u >= U1), len(mine))
        assert all(u < U1 for u in mine[:first_down]) and all(u >= U1 for u in mine[first_down:])
        # every chunk this pair waits for has its gate/up units among units that
        # some pair reaches before any of its own down units
        for u in mine[first_down:]:
            q = down[u - U1]
            assert all(v < U1 for v, qq in up.items() if qq == q)
