"""The FP4 indexer (fp8_fp4_mqa_logits) on the GPU, through the C ABI,
against the oracle.

Every entry is compared on small and ragged shapes (several head counts,
head dims, key counts that are not multiples of the 128-key tile, ranges that
are empty, negative or past the end); the bench-sized workloads on sampled
query rows.  Bound: |dlogit| <= (D + Hh) * 2^-23 * sum_h |w_h| sum_d |q_d k_d|
(FP32 accumulation of D products and Hh weighted terms, with a factor 2 of
slack); the -inf entries must sit exactly where the oracle puts them, and
without cleaning nothing outside the ranges may be written.
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _run(d, clean=True, sentinel=None):
    import torch

    import block_scaled_fp8_permute_b200 as moe
    S, Hh, D = d["q"].shape
    N = d["kv"].shape[0]
    dev = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in d.items()}
    out = torch.full((max(S, 1), max(N, 1)), float("nan") if sentinel is None else sentinel,
                     dtype=torch.float32, device="cuda")
    ws = moe.alloc_mqa_workspace(S, Hh, D, N, "cuda")
    moe.moe_fp8_fp4_mqa_logits(dev["q"], dev["q_sf"], dev["kv"], dev["kv_sf"], dev["weights"],
                               dev["ks"], dev["ke"], out, ws, clean=clean)
    torch.cuda.synchronize()
    return out[:S, :N].cpu().numpy(), moe.moe_get_device_status(ws)


def _check(got, d, rows=None, label=""):
    S, Hh, D = d["q"].shape
    sub = dict(d)
    if rows is not None:
        for k in ("q", "q_sf", "weights", "ks", "ke"):
            sub[k] = np.ascontiguousarray(d[k][rows])
        got = got[rows]
    ref, mag = oracle.mqa_logits(**sub, want_mag=True)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref)), label
    fin = np.isfinite(ref)
    assert np.isfinite(got[fin]).all(), label
    tol = (D + Hh) * 2.0 ** -23 * mag[fin] + 1e-30
    err = np.abs(got[fin].astype(np.float64) - ref[fin])
    assert (err <= tol).all(), (label, float((err / tol).max()))
    return float((err / np.maximum(tol, 1e-300)).max()) if err.size else 0.0


def _inputs(S, Hh, D, N, seed):
    d = synth.make_indexer(S, Hh, D, N, seed)
    rng = np.random.default_rng(seed)
    d["ks"] = rng.integers(-5, max(N, 1), S).astype(np.int32)
    d["ke"] = (d["ks"] + rng.integers(-3, N + 40, S)).astype(np.int32)
    d["ks"][0], d["ke"][0] = 0, N                 # one full row
    if S > 1:
        d["ks"][1], d["ke"][1] = 7, 3             # one empty row
    return d


@pytest.mark.parametrize("S,Hh,D,N", [
    (5, 64, 128, 300),      # one query group, 3 key tiles (last one partial)
    (33, 32, 256, 129),     # 2 K-blocks, 5 groups of 8 tokens, 129 keys
    (9, 128, 128, 64),      # 2 tokens per group, fewer keys than one tile
    (40, 16, 384, 1000),    # 16 tokens per group, 3 K-blocks
    (1, 64, 128, 1),        # one query, one key
])
def test_small_shapes_every_entry(S, Hh, D, N):
    d = _inputs(S, Hh, D, N, seed=S + N)
    got, st = _run(d)
    assert st == 0
    _check(got, d, label=f"S{S} Hh{Hh} D{D} N{N}")


@pytest.mark.parametrize("S,Hh,D,N,sms", [
    (40, 16, 384, 1000, 3),   # 3 CTAs: several two-tile units and group changes each
    (20, 64, 128, 700, 1),    # one CTA walks every tile: query slots and key ring wrap
    (33, 32, 256, 129, 2),    # 2 K-blocks: seven key stages
    (9, 128, 512, 400, 1),    # 4 K-blocks: a single query slot
    (7, 64, 1024, 300, 2),    # 8 K-blocks: one query slot, one key stage
    (6, 128, 128, 2000, 1),   # 128 heads: one token per tile, two TMEM load chunks per warp
    (14, 32, 128, 900, 2),    # 32 heads: six tokens per tile, two per epilogue warp
])
def test_few_ctas_many_tiles_each(S, Hh, D, N, sms):
    """With the SM count capped, every CTA runs many tiles and query groups,
    so the query slots, their scale buffers and the key ring are reused."""
    import block_scaled_fp8_permute_b200 as moe
    d = _inputs(S, Hh, D, N, seed=S * 7 + N)
    moe.moe_set_num_sms(sms)
    try:
        got, st = _run(d)
    finally:
        moe.moe_set_num_sms(0)
    assert st == 0
    _check(got, d, label=f"S{S} Hh{Hh} D{D} N{N} sms{sms}")


def test_without_cleaning_nothing_outside_the_ranges_is_written():
    d = _inputs(12, 64, 128, 500, seed=3)
    got, st = _run(d, clean=False, sentinel=12345.0)
    assert st == 0
    ref, _ = oracle.mqa_logits(**d)
    outside = np.isneginf(ref)
    assert (got[outside] == 12345.0).all()
    _check(np.where(outside, -np.inf, got), d, label="unclean")


def test_deterministic_and_prefix_ranges():
    d = synth.make_indexer(20, 64, 128, 700, seed=9)
    a, _ = _run(d)
    b, _ = _run(d)
    assert np.array_equal(a, b)
    _check(a, d, label="prefix")


@pytest.mark.parametrize("name", ["indexer", "indexer-decode"])
def test_bench_workloads_sampled_rows(name):
    wl = synth.INDEXER_WORKLOADS[name]
    d = synth.make_indexer(wl.S, wl.Hh, wl.D, wl.N, wl.seed)
    got, st = _run(d)
    assert st == 0
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([[0, wl.S - 1], rng.choice(wl.S, min(6, wl.S), replace=False)]))
    _check(got, d, rows=rows, label=name)
