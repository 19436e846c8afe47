"""End-to-end parity of the MoE layer forward on the GPU (through the C ABI)
against the CPU oracle.

Small and ragged shapes are compared on every token; the full-size
workloads (the launch configuration bench.py times) on a sample of tokens
the oracle computes one by one.  Bound: normwise relative error <= 5e-3 and
per element |dy| <= 2e-2 * (|y_ref| + rms(y_ref)); invariants that hold at
any size (token permutation, determinism, the host-buffer entry point) are
checked bit-exactly.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import Layer, assert_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _inputs(T, H, I, E, k, seed=0, mode=0, zipf=0.0):
    x, x_sf = synth.make_x(T, H, seed)
    w1, w1_sf = synth.make_w(E, 2 * I, H, 2, seed)
    w2, w2_sf = synth.make_w(E, H, I, 3, seed)
    idx, tw = synth.make_routing(T, E, k, mode, zipf, seed)
    return dict(x=x, x_sf=x_sf, topk_idx=idx, topk_w=tw, w1=w1, w1_sf=w1_sf, w2=w2, w2_sf=w2_sf)


def _check_full(inputs, label):
    lay = Layer(inputs).run()
    y = lay.y_bits()
    y_ref, _, bad = oracle.moe_forward(**inputs)
    p = assert_parity(y, y_ref, label)
    assert lay.status() == (6 if bad else 0)
    return lay, p


def test_tiny_workload_all_tokens(gemm_variant):
    _check_full(synth.make_inputs(synth.workload("tiny")), "tiny")


@pytest.fixture(params=[(0, 64, -1), (0, 0, -1), (0, 0, 1), (0, 0, 0), (1, 64, -1), (1, 0, -1)],
                ids=["one-sm+swap", "one-sm", "one-sm+narrow", "one-sm-no-narrow",
                     "sm-pair+swap", "sm-pair"])
def gemm_variant(request):
    """Tiling of the normal GEMM tiles x the swapped-role threshold (0: every
    expert uses normal tiles; 64: experts with <= 64 rows use swapped roles) x
    the narrow-tile mode (-1 auto, 1 forced on, 0 off)."""
    import block_scaled_fp8_permute_b200 as moe
    variant, swap_max, narrow = request.param
    moe.moe_set_gemm_variant(variant)
    moe.moe_set_swap_max(swap_max)
    moe.moe_set_narrow_tiles(narrow)
    yield request.param
    moe.moe_set_gemm_variant(0)
    moe.moe_set_swap_max(0)
    moe.moe_set_narrow_tiles(-1)


@pytest.mark.parametrize("T,H,I,E,k", [
    (1, 256, 256, 4, 2),       # one token
    (37, 128, 128, 5, 3),      # H = 128: linear2 runs a half-width (128-column) tile
    (300, 384, 256, 16, 4),    # H = 384: one full and one half tile along N
    (130, 256, 384, 3, 3),     # m-tile tail: 130*3 rows over 3 experts
    (200, 512, 128, 64, 6),    # many experts, some empty
    (600, 384, 256, 40, 3),    # mixed: experts above and below the swap threshold
    (90, 256, 256, 2, 1),      # 45-ish rows per expert: swapped tiles of N = 48
])
def test_ragged_shapes_all_tokens(T, H, I, E, k, gemm_variant):
    _check_full(_inputs(T, H, I, E, k, seed=T + H), f"T{T}H{H}I{I}E{E}k{k}")


def test_unused_slots_duplicates_and_bad_ids(gemm_variant):
    d = _inputs(96, 256, 256, 6, 4, seed=5)
    idx = d["topk_idx"].copy()
    idx[::7, 1] = -1                 # unused slots
    idx[::5, 2] = idx[::5, 0]        # the same expert twice in one token
    idx[3, 3] = 6                    # invalid id: skipped, reported
    idx[10, 0] = -9
    d["topk_idx"] = idx
    lay, _ = _check_full(d, "slots")
    assert lay.status() == 6


@pytest.mark.parametrize("plan_variant,fwd_variant", [(0, 1), (1, 0)])
def test_tiling_switched_between_plan_and_forward(plan_variant, fwd_variant):
    """Many small experts (narrow tiles with one-SM tiling): the plan made with
    one tiling variant, the forward run with the other, still computes every row."""
    import block_scaled_fp8_permute_b200 as moe
    d = _inputs(200, 512, 128, 64, 6, seed=4)
    try:
        moe.moe_set_gemm_variant(plan_variant)
        lay = Layer(d)
        moe.moe_plan(lay.shape, lay.dev["topk_idx"], lay.ws)
        moe.moe_set_gemm_variant(fwd_variant)
        dv = lay.dev
        moe.moe_forward(lay.shape, dv["x"], dv["x_sf"], dv["topk_idx"], dv["topk_w"], *lay.wt,
                        lay.y, lay.ws)
        y = lay.y_bits()
    finally:
        moe.moe_set_gemm_variant(0)
    y_ref, _, _ = oracle.moe_forward(**d)
    assert_parity(y, y_ref, f"plan {plan_variant} forward {fwd_variant}")
    assert lay.status() == 0


@pytest.mark.parametrize("knob,plan_value,fwd_value", [
    ("narrow", 1, 0), ("narrow", 0, 1), ("narrow", -1, 0), ("swap", 64, 0), ("swap", 0, 64)])
def test_knob_changed_between_plan_and_forward(knob, plan_value, fwd_value):
    """The plan moves small experts to narrow or swapped-role tiles according
    to the knobs' values at plan time; changing a knob before the forward must
    not drop those experts' rows (status stays 0, y matches the oracle)."""
    import block_scaled_fp8_permute_b200 as moe
    d = _inputs(200, 512, 128, 64, 6, seed=11)   # ~19 rows per expert
    setter = moe.moe_set_narrow_tiles if knob == "narrow" else moe.moe_set_swap_max
    default = -1 if knob == "narrow" else 0
    try:
        setter(plan_value)
        lay = Layer(d)
        moe.moe_plan(lay.shape, lay.dev["topk_idx"], lay.ws)
        setter(fwd_value)
        dv = lay.dev
        moe.moe_forward(lay.shape, dv["x"], dv["x_sf"], dv["topk_idx"], dv["topk_w"], *lay.wt,
                        lay.y, lay.ws)
        y = lay.y_bits()
    finally:
        setter(default)
    y_ref, _, _ = oracle.moe_forward(**d)
    assert_parity(y, y_ref, f"{knob} {plan_value} -> {fwd_value}")
    assert lay.status() == 0


def test_all_rows_one_expert_and_empty_experts():
    d = _inputs(200, 256, 256, 8, 2, seed=9)
    d["topk_idx"][:, 0] = 3
    d["topk_idx"][:, 1] = 5
    _check_full(d, "two-experts")


def test_token_permutation_and_determinism():
    d = synth.make_inputs(synth.workload("tiny"))
    lay = Layer(d).run()
    y1 = lay.y_bits()
    y1b = lay.run().y_bits()
    assert np.array_equal(y1, y1b)                       # run to run
    perm = np.random.default_rng(3).permutation(d["x"].shape[0])
    d2 = dict(d)
    for key in ("x", "x_sf", "topk_idx", "topk_w"):
        d2[key] = np.ascontiguousarray(d[key][perm])
    y2 = Layer(d2).run().y_bits()
    assert np.array_equal(y2, y1[perm])                  # rows are independent


def test_host_buffer_entry_point_matches_device_entry_point():
    import torch

    import block_scaled_fp8_permute_b200 as moe
    d = synth.make_inputs(synth.workload("tiny"))
    lay = Layer(d).run()
    y_dev = lay.y_bits()
    ws = moe.alloc_workspace(lay.shape, "cuda", host_variant=True)
    pin = {k: torch.from_numpy(np.ascontiguousarray(d[k])).pin_memory()
           for k in ("x", "x_sf", "topk_idx", "topk_w")}
    y_host = torch.empty(d["x"].shape, dtype=torch.int16).pin_memory()
    moe.moe_forward_host(lay.shape, pin["x"], pin["x_sf"], pin["topk_idx"], pin["topk_w"],
                         *lay.wt, y_host, ws)
    assert np.array_equal(y_host.numpy().view(np.uint16), y_dev)


def test_pipelined_host_entry_point_matches_per_batch_results():
    """Five batches (three distinct inputs, reused so both staging slots are
    recycled) through the overlapped host-buffer call: each y equals the
    device entry point's result for its inputs, bit for bit."""
    import torch

    import block_scaled_fp8_permute_b200 as moe
    d = synth.make_inputs(synth.workload("tiny"))
    T = d["x"].shape[0]
    perm = np.random.default_rng(11).permutation(T)
    d_b = dict(d)
    for key in ("x", "x_sf", "topk_idx", "topk_w"):
        d_b[key] = np.ascontiguousarray(d[key][perm])
    d_c = dict(d)
    d_c["topk_idx"] = np.ascontiguousarray(np.roll(d["topk_idx"], 1, axis=1))  # other routing
    lay = Layer(d).run()
    expect = [lay.y_bits(), lay.y_bits()[perm], Layer(d_c).run().y_bits()]
    pins = []
    for src in (d, d_b, d_c):
        pins.append({k: torch.from_numpy(np.ascontiguousarray(src[k])).pin_memory()
                     for k in ("x", "x_sf", "topk_idx", "topk_w")})
    order = [0, 1, 2, 0, 1]
    ys = [torch.full(d["x"].shape, -1, dtype=torch.int16).pin_memory() for _ in order]
    ws = moe.alloc_workspace(lay.shape, "cuda", host_variant="pipelined")
    assert ws.numel() > moe.moe_workspace_bytes_host(lay.shape)
    moe.moe_forward_host_pipelined(lay.shape, [pins[b]["x"] for b in order],
                                   [pins[b]["x_sf"] for b in order],
                                   [pins[b]["topk_idx"] for b in order],
                                   [pins[b]["topk_w"] for b in order], *lay.wt, ys, ws)
    for i, b in enumerate(order):
        assert np.array_equal(ys[i].numpy().view(np.uint16), expect[b]), f"batch {i}"
    assert moe.moe_get_device_status(ws) == 0


_WEIGHTS = {}


def _full_inputs(wl):
    """Full-size inputs; the weights of workloads sharing a layer shape are
    generated once per session (skewed and decode share theirs)."""
    key = (wl.E, wl.H, wl.I, wl.seed)
    if key not in _WEIGHTS:
        _WEIGHTS.clear()
        _WEIGHTS[key] = synth.make_weights(wl)
    x, x_sf, idx, tw = synth.make_activations(wl)
    w1, w1_sf, w2, w2_sf = _WEIGHTS[key]
    return dict(x=x, x_sf=x_sf, topk_idx=idx, topk_w=tw, w1=w1, w1_sf=w1_sf, w2=w2, w2_sf=w2_sf)


@pytest.fixture(params=[(0, 0, -1), (0, 0, 0), (0, 64, -1), (1, 0, -1)],
                ids=["default", "no-narrow", "swap", "sm-pair"])
def full_variant(request):
    import block_scaled_fp8_permute_b200 as moe
    variant, swap_max, narrow = request.param
    moe.moe_set_gemm_variant(variant)
    moe.moe_set_swap_max(swap_max)
    moe.moe_set_narrow_tiles(narrow)
    yield request.param
    moe.moe_set_gemm_variant(0)
    moe.moe_set_swap_max(0)
    moe.moe_set_narrow_tiles(-1)


@pytest.mark.parametrize("name,n_sample", [
    ("mid", 96), ("usage", 12), ("skewed", 24), ("decode", 48), ("decode@T16", 16),
    ("decode@T32", 32), ("decode@T64", 32),
])
def test_full_size_sampled(name, n_sample, full_variant):
    """Full-size workloads in the launch configuration bench.py uses; the
    oracle computes a seeded sample of tokens (first, last, random)."""
    wl = synth.workload(name)
    d = _full_inputs(wl)
    lay = Layer(d).run()
    y = lay.y_bits()
    assert lay.status() == 0
    rng = np.random.default_rng(1)
    toks = np.unique(np.concatenate([[0, wl.T - 1], rng.choice(wl.T, n_sample, replace=False)]))
    y_ref, _, _ = oracle.moe_forward(**d, tokens=toks.astype(np.int32))
    assert_parity(y[toks], y_ref, name)
    # every output finite, nothing left unwritten
    assert np.isfinite((y.astype(np.uint32) << 16).view(np.float32)).all()
