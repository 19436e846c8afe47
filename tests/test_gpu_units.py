"""GPU unit parity through the C ABI: plan indices (bit-exact against the
oracle's counting sort), weight transform (bit-exact round trip), and the
epilogue requantiser (bit-exact codes and scales on identical FP32 inputs)."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_scaled_fp8_permute_b200 as m
    return m


def _gpu_plan(moe, idx: np.ndarray, E: int):
    import torch
    T, k = idx.shape
    shp = moe.shape(T, 256, 256, E, k)
    ws = moe.alloc_workspace(shp, "cuda")
    d_idx = torch.from_numpy(np.ascontiguousarray(idx)).cuda()
    moe.moe_plan(shp, d_idx, ws)
    return moe.moe_plan_export(shp, ws), moe.moe_get_device_status(ws)


def _routings():
    cases = []
    for name in ("tiny", "mid", "skewed", "decode", "decode@T16", "usage"):
        wl = synth.workload(name)
        idx, _ = synth.make_routing(wl.T, wl.E, wl.k, wl.mode, wl.zipf_s, wl.seed)
        cases.append((name, idx, wl.E))
    rng = np.random.default_rng(7)
    idx = rng.integers(0, 5, (37, 3)).astype(np.int32)
    idx[rng.random((37, 3)) < 0.2] = -1
    cases.append(("ragged-unused-slots", idx, 5))
    cases.append(("one-token", np.array([[3, 0]], np.int32), 4))
    cases.append(("all-one-expert", np.zeros((300, 2), np.int32), 8))   # duplicates in a token
    idx = rng.integers(0, 1024, (2500, 8)).astype(np.int32)
    cases.append(("E1024", idx, 1024))
    idx = rng.integers(0, 64, (8192, 8)).astype(np.int32)                 # R = 65536
    cases.append(("R65536", idx, 64))
    return cases


@pytest.mark.parametrize("case", _routings(), ids=lambda c: c[0])
def test_plan_bit_exact(moe, case):
    name, idx, E = case
    got, status = _gpu_plan(moe, idx, E)
    ref = oracle.plan(idx, E, moe.moe_block_m())
    assert status == 0
    assert got["P"] == ref["P"]
    for key in ("counts", "offs", "poffs", "row_of", "src_of"):
        assert np.array_equal(got[key], ref[key]), key


def test_plan_reports_bad_ids(moe):
    idx = np.array([[0, 9], [1, -1], [-7, 2]], np.int32)
    got, status = _gpu_plan(moe, idx, 4)
    ref = oracle.plan(idx, 4, 128)
    assert status == 6                                   # MOE_ERR_BAD_EXPERT_ID
    assert np.array_equal(got["row_of"], ref["row_of"])
    assert np.array_equal(got["src_of"], ref["src_of"])


def _inverse_transform(wt, wt_sf, E, N, K, interleave):
    """Host inverse of the documented transformed layout."""
    KB = K // 128
    codes = wt.reshape(E, KB, N, 64)
    w = np.empty((E, N, K // 2), np.uint8)
    sf = np.empty((E, N, K // 32), np.uint8)
    n = np.arange(N)
    if interleave:
        g, j = n // 256, n % 256
        src = np.where(j < 128, g * 128 + j, N // 2 + g * 128 + (j - 128))
    else:
        src = n
    chunks = wt_sf.reshape(E, KB, N // 128, 512)
    r = n % 128
    off = (r % 32) * 16 + (r // 32) * 4
    for kb in range(KB):
        w[:, src, kb * 64:(kb + 1) * 64] = codes[:, kb, :, :]
        for j4 in range(4):
            sf[:, src, kb * 4 + j4] = chunks[:, kb, n // 128, off + j4]
    return w, sf


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_transform_round_trip(moe, name):
    import torch
    wl = synth.workload(name)
    w1, w1_sf, w2, w2_sf = synth.make_weights(wl)
    shp = moe.shape(wl.T, wl.H, wl.I, wl.E, wl.k)
    d = [torch.from_numpy(a).cuda() for a in (w1, w1_sf, w2, w2_sf)]
    outs = moe.transform_weights(shp, *d)
    torch.cuda.synchronize()
    h = [o.cpu().numpy() for o in outs]
    r1, r1sf = _inverse_transform(h[0], h[1], wl.E, 2 * wl.I, wl.H, True)
    r2, r2sf = _inverse_transform(h[2], h[3], wl.E, wl.H, wl.I, False)
    assert np.array_equal(r1, w1) and np.array_equal(r1sf, w1_sf)
    assert np.array_equal(r2, w2) and np.array_equal(r2sf, w2_sf)


def test_requant_bit_exact(moe):
    import torch
    rng = np.random.default_rng(11)
    rows, cols = 512, 256
    a = (rng.standard_normal((rows, cols)) * np.exp(rng.uniform(-20, 20, (rows, 1)))).astype(np.float32)
    a[0, :32] = 0.0
    a[1, :32] = np.float32(448.0)                       # amax exactly at the E4M3 max
    a[2, :32] = np.float32(448.0) * np.float32(1.0000001)
    a[3, :] = np.float32(1e-40)                          # subnormal amax
    a[4, :] = rng.uniform(-3e38, 3e38, cols).astype(np.float32)
    pos = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)  # ties of the E4M3 grid, scale 2^0
    a[5, :126] = mids[:126]
    a[5, 126:252] = -mids[:126]
    a[5, 252:] = 0.0
    for b in range(cols // 32):                           # pin each block's scale to 2^0
        a[5, 32 * b + 31] = 448.0
    codes_ref, sb_ref = oracle.requant_rows(a)
    d_a = torch.from_numpy(a).cuda()
    codes = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    sb = torch.empty((rows, cols // 32), dtype=torch.uint8, device="cuda")
    moe.moe_debug_requant(d_a, codes, sb)
    torch.cuda.synchronize()
    assert np.array_equal(sb.cpu().numpy(), sb_ref)
    assert np.array_equal(codes.cpu().numpy(), codes_ref)
