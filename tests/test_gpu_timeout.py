"""Failure detection without a GPU fault: a device wait that can never end is
reported, not hung on.

A test hook makes the linear1 kernel's producer skip the loads of one
pipeline iteration, so the MMA issuer's bounded wait for that stage expires
(its limit shortened to 1 ms).  The kernel must record MOE_ERR_TIMEOUT with
the MMA issuer's site, every role of the CTA must stop waiting and the
kernel must return with the context usable; the next normal forward on the
same workspace must match the oracle again.  (The pages' change list fixes a
kernel hang: "DeepSeek DeepGEMM 2026年4月重磅更新" section 1, and the
discuss.deepseek.club topic 1597 post.)"""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import Layer, assert_parity

pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = 5
SITE_MMA_LINEAR1 = 21


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


# tiny: H = 256, so every CTA of linear1 runs one tile of two 128-K iterations
@pytest.mark.parametrize("skip_iteration", [0, 1])
def test_expired_wait_is_reported_and_the_next_forward_is_correct(skip_iteration):
    import time

    import torch

    import block_scaled_fp8_permute_b200 as moe
    moe.moe_set_narrow_tiles(0)   # every expert on the normal one-SM tiles the hook sits in
    d = synth.make_inputs(synth.workload("tiny"))
    try:
        lay = Layer(d)
        moe.moe_debug_set_fault(skip_iteration, 1_000_000)   # 1 ms
        t0 = time.perf_counter()
        lay.run()
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        moe.moe_debug_set_fault(-1, 0)
        assert lay.status() == MOE_ERR_TIMEOUT
        assert moe.moe_get_timeout_site(lay.ws) == SITE_MMA_LINEAR1
        assert elapsed < 1.0          # bounded by the shortened limits, not the 2 s default
        # the context is still usable: a normal forward on the same workspace
        lay.run()
        y = lay.y_bits()
        assert lay.status() == 0
        assert moe.moe_get_timeout_site(lay.ws) == 0
    finally:
        moe.moe_debug_set_fault(-1, 0)
        moe.moe_set_narrow_tiles(-1)
    y_ref, _, _ = oracle.moe_forward(**d)
    assert_parity(y, y_ref, "after timeout")
    assert np.isfinite((y.astype(np.uint32) << 16).view(np.float32)).all()


SITE_MMA_INDEXER = {0: 120, 1: 121}   # the MMA thread of ring 0 / ring 1


@pytest.mark.parametrize("skip_tile", [0, 1])
def test_indexer_expired_wait_is_reported_and_the_next_call_is_correct(skip_tile):
    """The FP4 indexer's producer leaves the key stage of one active tile
    unfilled (tile 0 goes to the first MMA thread's ring, tile 1 to the
    second's); that thread's bounded wait expires, the call reports
    MOE_ERR_TIMEOUT with its site, and the next call on the same workspace
    matches the oracle."""
    import time

    import torch

    import block_scaled_fp8_permute_b200 as moe
    from tests.test_gpu_indexer import _check, _inputs

    d = _inputs(20, 64, 128, 700, seed=5)
    S, Hh, D = d["q"].shape
    N = d["kv"].shape[0]
    dev = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in d.items()}
    out = torch.full((S, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = moe.alloc_mqa_workspace(S, Hh, D, N, "cuda")

    def call():
        moe.moe_fp8_fp4_mqa_logits(dev["q"], dev["q_sf"], dev["kv"], dev["kv_sf"], dev["weights"],
                                   dev["ks"], dev["ke"], out, ws)
    moe.moe_set_num_sms(2)   # two CTAs, about twenty tiles each
    try:
        moe.moe_debug_set_fault(skip_tile, 1_000_000)   # 1 ms
        t0 = time.perf_counter()
        call()
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        moe.moe_debug_set_fault(-1, 0)
        assert moe.moe_get_device_status(ws) == MOE_ERR_TIMEOUT
        assert moe.moe_get_timeout_site(ws) == SITE_MMA_INDEXER[skip_tile]
        assert elapsed < 1.0
        call()
        torch.cuda.synchronize()
        assert moe.moe_get_device_status(ws) == 0
        assert moe.moe_get_timeout_site(ws) == 0
        _check(out.cpu().numpy(), d, label=f"after timeout, skip {skip_tile}")
    finally:
        moe.moe_debug_set_fault(-1, 0)
        moe.moe_set_num_sms(0)
