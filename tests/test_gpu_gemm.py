"""The tcgen05 GEMM core (through the C-ABI test hooks) against float64
products on the CPU, over several tiles, ragged tails, split K and grouped
(mixture-of-experts) schedules with empty groups and multi-pass groups, on
single CTAs and on CTA pairs (tcgen05.mma.cta_group::2)."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _bf16(rng, shape, scale=1.0):
    x = torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32)).to(torch.bfloat16)
    return x


def _ref(a, b):
    return a.double().numpy() @ b.double().numpy().T


@pytest.fixture(scope="module")
def dg():
    import discrete_diffusion_moe_b200 as m
    return m


@pytest.mark.parametrize("M,N,K,ks", [(128, 16, 64, 1), (256, 256, 512, 1), (384, 200, 320, 1),
                                      (256, 600, 2816, 1), (128, 256, 1024, 4), (640, 48, 704, 3),
                                      # more units than SMs: several tiles per persistent CTA,
                                      # both accumulator buffers and stage-ring wrap-around
                                      (128 * 300, 32, 640, 1), (128 * 40, 1024, 256, 2)])
def test_dense_gemm(dg, M, N, K, ks):
    rng = np.random.default_rng(M * 7 + N + K)
    a, b = _bf16(rng, (M, K)), _bf16(rng, (N, K))
    da, db = a.cuda(), b.cuda()
    dd = torch.full((ks, M, N), float("nan"), device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    dg.check(dg.dg_test_gemm(da.data_ptr(), M, db.data_ptr(), N, K, dd.data_ptr(), ks, st))
    got = dd.sum(0).double().cpu().numpy()
    ref = _ref(a, b)
    # fp32 accumulation of exact bf16 products: error ~ sqrt(K) * 2^-24 * |a||b|
    tol = 1e-5 * np.sqrt(K) * 4 + 1e-6
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= tol * np.abs(ref).max() + 1e-4, np.abs(got - ref).max()


@pytest.mark.parametrize("bn,sizes,R", [(16, [17, 0, 43, 1, 90, 5], 256), (32, [17, 0, 43, 1, 90, 5], 256),
                                        (64, [17, 0, 43, 1, 90, 5], 256), (256, [17, 0, 43, 1, 90, 5], 256),
                                        # skewed routing: one group holds most rows
                                        (64, [3, 600, 0, 0, 9, 300], 256),
                                        # CTA pairs: an odd tile count (the last pair's second tile
                                        # is missing), a partial second tile, every B box size
                                        (128, [17, 0, 43, 1, 90, 5], 384), (32, [33, 64, 0, 7], 200),
                                        (16, [1, 2, 3, 15, 16, 17, 31, 33], 256)])
def test_grouped_gemm(dg, bn, sizes, R):
    rng = np.random.default_rng(bn + len(sizes) + sizes[1] + R)
    G, K = len(sizes), 192
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    n = int(off[-1])
    a, b = _bf16(rng, (G * R, K)), _bf16(rng, (n, K))
    dd = torch.full((n, R), float("nan"), device="cuda")
    doff = torch.from_numpy(off).cuda()
    da, db = a.cuda(), b.cuda()  # keep the device copies alive across the call
    choff = torch.zeros(G + 1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    dg.check(dg.dg_test_grouped_gemm(da.data_ptr(), R, G, db.data_ptr(), n, K, doff.data_ptr(),
                                     dd.data_ptr(), bn, choff.data_ptr(), st))
    got = dd.double().cpu().numpy()
    A = a.double().numpy().reshape(G, R, K)
    B = b.double().numpy()
    for g in range(G):
        rows = slice(off[g], off[g + 1])
        ref = B[rows] @ A[g].T
        if sizes[g]:
            assert np.abs(got[rows] - ref).max() <= 1e-4 * max(1.0, np.abs(ref).max()), g


def test_gemm_rejects_bad_shapes(dg):
    with pytest.raises(dg.DgError):
        dg.check(dg.dg_test_gemm(None, 128, None, 16, 64, None, 1, None))


@pytest.mark.parametrize("M,N,K,ks,mt,bn", [(256, 256, 512, 1, 2, 256), (384, 200, 320, 1, 2, 256),
                                          (128 * 23, 256, 1024, 3, 2, 256), (128 * 45, 256, 2816, 3, 2, 128),
                                          (640, 48, 704, 2, 2, 64), (128 * 300, 32, 640, 1, 2, 32)])
def test_dense_gemm_two_a_tiles(dg, M, N, K, ks, mt, bn):
    """Units of two 128-row A tiles (one B tile feeding two MMAs): odd tile
    counts (a last unit with one tile), one or two accumulator buffers."""
    rng = np.random.default_rng(M + N + K + mt)
    a, b = _bf16(rng, (M, K)), _bf16(rng, (N, K))
    da, db = a.cuda(), b.cuda()
    dd = torch.full((ks, M, N), float("nan"), device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    dg.check(dg.lib.dg_test_gemm_tiles(da.data_ptr(), M, db.data_ptr(), N, K, dd.data_ptr(), ks, mt, bn, st))
    got = dd.sum(0).double().cpu().numpy()
    ref = _ref(a, b)
    tol = 1e-5 * np.sqrt(K) * 4 + 1e-6
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= tol * np.abs(ref).max() + 1e-4, np.abs(got - ref).max()
