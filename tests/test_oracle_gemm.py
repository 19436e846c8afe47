"""Pins for the oracle's FP8 x FP4 GEMM (dense and masked grouped).

The oracle's GEMM is compared with an independently written numpy formulation
(tests/independent_ref.py: vectorised decodes, a dense matmul in float64 and
its own bf16 rounding), with a closed form, and with the masked layout's
contract (rows at and past a group's count are left alone).
"""
import numpy as np
import pytest

import independent_ref as ind
import oracle
import synth


def _inputs(G, M, N, K, seed):
    a, a_sf = synth.make_x(G * M, K, seed)
    b, b_sf = synth.make_w(G, N, K, 2, seed)
    return a.reshape(G, M, K), a_sf.reshape(G, M, K // 128), b, b_sf


def _numpy_gemm(a, a_sf, b, b_sf):
    G = a.shape[0]
    out = []
    for g in range(G):
        A = ind.dequant_x(a[g], a_sf[g])
        B = ind.dequant_w(b[g:g + 1], b_sf[g:g + 1])[0]
        out.append(ind.bf16_value(A @ B.T))
    return np.stack(out)


def _bits_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("G,M,N,K", [(1, 7, 128, 128), (1, 33, 256, 384), (3, 20, 128, 256)])
def test_gemm_matches_numpy_formulation(G, M, N, K):
    a, a_sf, b, b_sf = _inputs(G, M, N, K, seed=G + M + N + K)
    d = oracle.gemm(a, a_sf, b, b_sf)
    ref = _numpy_gemm(a, a_sf, b, b_sf)
    got = _bits_to_f64(d)
    # double sums in another order: identical bf16 results except, at most, a
    # value lying on a rounding boundary to within the summation error
    exact = (got == ref).mean()
    assert exact > 0.999, exact
    ulp = np.abs(ref) * 2.0 ** -7 + 1e-30
    assert (np.abs(got - ref) <= ulp).all()


def test_gemm_dense_equals_single_group():
    a, a_sf, b, b_sf = _inputs(1, 17, 128, 256, seed=5)
    d2 = oracle.gemm(a[0], a_sf[0], b[0], b_sf[0])
    d3 = oracle.gemm(a, a_sf, b, b_sf)
    assert np.array_equal(d2, d3[0])


def test_gemm_closed_form():
    """A = 1.0 everywhere (E4M3 0x38, scale byte 127), B = 0.5 (E2M1 0x1) with
    scale byte 126 (x 0.5): every output is K * 1.0 * 0.25 = K / 4, exact in bf16."""
    M, N, K = 4, 128, 256
    a = np.full((M, K), 0x38, np.uint8)
    a_sf = np.full((M, K // 128), 0x7F7F7F7F, np.int32)
    b = np.full((N, K // 2), 0x11, np.uint8)
    b_sf = np.full((N, K // 32), 126, np.uint8)
    d = oracle.gemm(a, a_sf, b, b_sf)
    assert np.all(_bits_to_f64(d) == K / 4)


def test_gemm_masked_rows_left_alone():
    G, M, N, K = 3, 40, 128, 128
    a, a_sf, b, b_sf = _inputs(G, M, N, K, seed=9)
    masked = np.array([0, 17, 40], np.int32)
    sentinel = np.full((G, M, N), 0x7FC1, np.uint16)
    d = oracle.gemm(a, a_sf, b, b_sf, masked_m=masked, out=sentinel)
    full = oracle.gemm(a, a_sf, b, b_sf)
    for g in range(G):
        c = masked[g]
        assert np.array_equal(d[g, :c], full[g, :c])
        assert np.all(d[g, c:] == 0x7FC1)
