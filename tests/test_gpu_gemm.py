"""The standalone FP8 x FP4 GEMM (dense and masked grouped) against the
oracle, through the C ABI."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import block_scaled_fp8_permute_b200 as moe
    return moe, torch


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _check(got_bits, ref_bits):
    if got_bits.size == 0:
        return
    got, ref = _f64(got_bits), _f64(ref_bits)
    assert np.isfinite(got).all()
    # FP32 accumulation on the GPU vs double in the oracle, one BF16 rounding
    # each: equal except where the sum lies within the FP32 error of a
    # rounding boundary, and then one BF16 step apart
    assert (got == ref).mean() > 0.995, (got == ref).mean()
    step = np.abs(ref) * 2.0 ** -7 + 1e-30
    assert (np.abs(got - ref) <= step).all()


def _gemm_inputs(G, M, N, K, seed):
    a, a_sf = synth.make_x(G * M, K, seed)
    b, b_sf = synth.make_w(G, N, K, 2, seed)
    return a.reshape(G, M, K), a_sf.reshape(G, M, K // 128), b, b_sf


def _dev(torch, arr):
    return torch.from_numpy(np.ascontiguousarray(arr)).cuda()


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (100, 256, 256), (300, 384, 512),
                                   (129, 128, 1024), (640, 512, 384)])
def test_dense_gemm_matches_oracle(env, M, N, K):
    moe, torch = env
    a, a_sf, b, b_sf = _gemm_inputs(1, M, N, K, seed=M + N + K)
    b_t, b_sf_t = moe.gemm_transform_b(1, N, K, _dev(torch, b), _dev(torch, b_sf))
    d = torch.full((M, N), 0x7FC1, dtype=torch.int16, device="cuda")
    ws = moe.alloc_gemm_workspace(1, M, N, K, "cuda")
    moe.moe_gemm_fp8_fp4(M, N, K, _dev(torch, a[0]), _dev(torch, a_sf[0]), b_t, b_sf_t, d, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    got = d.cpu().numpy().view(np.uint16)
    ref = oracle.gemm(a[0], a_sf[0], b[0], b_sf[0])
    _check(got, ref)


def test_masked_gemm_matches_oracle_and_leaves_rows(env):
    moe, torch = env
    G, M, N, K = 4, 256, 256, 384
    a, a_sf, b, b_sf = _gemm_inputs(G, M, N, K, seed=11)
    masked = np.array([0, 130, 256, 1], np.int32)
    b_t, b_sf_t = moe.gemm_transform_b(G, N, K, _dev(torch, b), _dev(torch, b_sf))
    d = torch.full((G, M, N), 0x7FC1, dtype=torch.int16, device="cuda")
    ws = moe.alloc_gemm_workspace(G, M, N, K, "cuda")
    mm = _dev(torch, masked)
    moe.moe_gemm_fp8_fp4_masked(G, M, N, K, _dev(torch, a), _dev(torch, a_sf), mm, b_t, b_sf_t,
                                d, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    got = d.cpu().numpy().view(np.uint16)
    ref = oracle.gemm(a, a_sf, b, b_sf, masked_m=masked,
                      out=np.full((G, M, N), 0x7FC1, np.uint16))
    for g in range(G):
        c = masked[g]
        _check(got[g, :c], ref[g, :c])
        assert np.all(got[g, c:] == 0x7FC1)


def test_masked_counts_out_of_range_reported(env):
    moe, torch = env
    G, M, N, K = 2, 128, 128, 128
    a, a_sf, b, b_sf = _gemm_inputs(G, M, N, K, seed=3)
    b_t, b_sf_t = moe.gemm_transform_b(G, N, K, _dev(torch, b), _dev(torch, b_sf))
    d = torch.zeros((G, M, N), dtype=torch.int16, device="cuda")
    ws = moe.alloc_gemm_workspace(G, M, N, K, "cuda")
    mm = _dev(torch, np.array([129, -5], np.int32))
    moe.moe_gemm_fp8_fp4_masked(G, M, N, K, _dev(torch, a), _dev(torch, a_sf), mm, b_t, b_sf_t,
                                d, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 1  # MOE_ERR_INVALID_ARG, counts clamped
    got = d.cpu().numpy().view(np.uint16)
    ref = oracle.gemm(a, a_sf, b, b_sf, masked_m=np.array([128, 0], np.int32))
    _check(got[0], ref[0])
    assert np.all(got[1] == 0)


def test_masked_gemm_follows_counts_in_a_cuda_graph(env):
    """The counts are read on the device: one captured graph, replayed with
    new counts written into the same buffer, computes the new row sets."""
    moe, torch = env
    G, M, N, K = 3, 128, 256, 256
    a, a_sf, b, b_sf = _gemm_inputs(G, M, N, K, seed=21)
    b_t, b_sf_t = moe.gemm_transform_b(G, N, K, _dev(torch, b), _dev(torch, b_sf))
    da, das = _dev(torch, a), _dev(torch, a_sf)
    d = torch.zeros((G, M, N), dtype=torch.int16, device="cuda")
    ws = moe.alloc_gemm_workspace(G, M, N, K, "cuda")
    mm = _dev(torch, np.array([5, 0, 128], np.int32))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        moe.moe_gemm_fp8_fp4_masked(G, M, N, K, da, das, mm, b_t, b_sf_t, d, ws,
                                    stream=s.cuda_stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        moe.moe_gemm_fp8_fp4_masked(G, M, N, K, da, das, mm, b_t, b_sf_t, d, ws,
                                    stream=s.cuda_stream)
    full = oracle.gemm(a, a_sf, b, b_sf)
    for counts in ([128, 77, 0], [1, 128, 64]):
        d.zero_()
        mm.copy_(torch.tensor(counts, dtype=torch.int32))
        graph.replay()
        torch.cuda.synchronize()
        got = d.cpu().numpy().view(np.uint16)
        for g, c in enumerate(counts):
            _check(got[g, :c], full[g, :c])
            assert np.all(got[g, c:] == 0)
    del graph


def test_dense_gemm_full_size_sampled_rows(env):
    """A prefill-sized GEMM (M=4096, N=K=7168): every tile runs, sampled rows
    checked against the oracle."""
    moe, torch = env
    M, N, K = 4096, 7168, 7168
    a, a_sf, b, b_sf = _gemm_inputs(1, M, N, K, seed=1)
    b_t, b_sf_t = moe.gemm_transform_b(1, N, K, _dev(torch, b), _dev(torch, b_sf))
    d = torch.empty((M, N), dtype=torch.int16, device="cuda")
    ws = moe.alloc_gemm_workspace(1, M, N, K, "cuda")
    moe.moe_gemm_fp8_fp4(M, N, K, _dev(torch, a[0]), _dev(torch, a_sf[0]), b_t, b_sf_t, d, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    rows = np.random.default_rng(0).choice(M, 12, replace=False)
    rows = np.concatenate([rows, [0, 127, 128, M - 1]])
    got = d.cpu().numpy().view(np.uint16)[rows]
    ref = oracle.gemm(a[0][rows], a_sf[0][rows], b[0], b_sf[0])
    _check(got, ref)
