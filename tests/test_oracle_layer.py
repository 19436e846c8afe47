"""Pins for the oracle's plan and layer forward.

Pinned by: hand-worked examples (tests/golden/hand_worked.txt), a dense FFN
special case and a masked all-experts formulation written independently in
numpy (tests/independent_ref.py), brute-force stable sorting, and
invariants (token permutation, slot permutation, weight doubling, poisoned
empty experts, unused slots).
"""
import os

import numpy as np
import pytest

import oracle
import synth
from tests import independent_ref as ind


# ------------------------------------------------------------------ plan
def _brute_plan(idx, E, bm):
    T, k = idx.shape
    flat = idx.reshape(-1)
    counts = np.array([(flat == e).sum() for e in range(E)], np.int32)
    poffs = np.concatenate([[0], np.cumsum((counts + bm - 1) // bm * bm)]).astype(np.int32)
    row_of = np.full(T * k, -1, np.int32)
    src_of = np.full(poffs[-1], -1, np.int32)
    for e in range(E):
        members = [i for i in range(T * k) if flat[i] == e]     # ascending = stable
        for r, i in enumerate(members):
            row_of[i] = poffs[e] + r
            src_of[poffs[e] + r] = i
    return counts, poffs, row_of, src_of


@pytest.mark.parametrize("T,k,E,bm", [(64, 2, 8, 128), (37, 3, 5, 16), (1, 1, 1, 128),
                                      (200, 8, 64, 128), (5, 2, 300, 128)])
def test_plan_matches_brute_force(T, k, E, bm):
    rng = np.random.default_rng(T * 100 + E)
    idx = rng.integers(0, E, (T, k)).astype(np.int32)
    idx[rng.random((T, k)) < 0.1] = -1
    p = oracle.plan(idx, E, bm)
    counts, poffs, row_of, src_of = _brute_plan(idx, E, bm)
    assert np.array_equal(p["counts"], counts)
    assert np.array_equal(p["poffs"], poffs)
    assert np.array_equal(p["offs"], np.concatenate([[0], np.cumsum(counts)]))
    assert np.array_equal(p["row_of"].reshape(-1), row_of)
    assert np.array_equal(p["src_of"], src_of)
    assert p["bad"] == 0
    # invariants
    valid = row_of >= 0
    assert counts.sum() == valid.sum()
    assert np.all(src_of[row_of[valid]] == np.nonzero(valid)[0])
    assert np.all(poffs % bm == 0)


def test_plan_counts_invalid_ids():
    idx = np.array([[0, 7], [-1, 2], [-5, 1]], np.int32)
    p = oracle.plan(idx, 4, 128)
    assert p["bad"] == 2
    assert list(p["counts"]) == [1, 1, 1, 0]
    assert p["row_of"][0, 1] == -1 and p["row_of"][2, 0] == -1


# ------------------------------------------------------------ hand-worked
def _read_cases(golden_dir):
    cases = {}
    with open(os.path.join(golden_dir, "hand_worked.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                parts = line.split()
                cases.setdefault(parts[0], {})[parts[1]] = [float(v) for v in parts[2:]]
    return cases


def _hand_inputs(case):
    H, I = 128, 32
    x = np.full((1, H), 0x38, np.uint8)
    x_sf = np.full((1, 1), 0x7F7F7F7F, np.int32)
    w1 = np.zeros((1, 2 * I, H), np.uint8)          # codes, one per element (packed below)
    w2 = np.zeros((1, H, I), np.uint8)
    w1_sf = np.full((1, 2 * I, H // 32), 127, np.uint8)
    w2_sf = np.full((1, H, I // 32), 127, np.uint8)
    tw = np.ones((1, 1), np.float32)
    if case in ("caseA", "caseB"):
        w1[0, :I, :] = 0x1
        w1[0, I:, :] = 0x2 if case == "caseA" else 0xA
        if case == "caseA":
            w2[:] = 0x2
        else:
            w2[:] = 0x3
            w2_sf[:] = 126
            tw[:] = 0.25
    else:
        x[:] = 0x00
        x[0, 0] = 0x38
        for j, c in enumerate([0x0, 0x1, 0x2, 0x7]):
            w1[0, j, 0] = c
        w1[0, I:, 0] = 0x2
        for n in range(4):
            w2[0, n, n] = 0x2

    def pack(codes):
        return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)

    return dict(x=x, x_sf=x_sf, topk_idx=np.zeros((1, 1), np.int32), topk_w=tw,
                w1=pack(w1), w1_sf=w1_sf, w2=pack(w2), w2_sf=w2_sf)


@pytest.mark.parametrize("case", ["caseA", "caseB", "caseC"])
def test_hand_worked_cases(golden_dir, case):
    spec = _read_cases(golden_dir)[case]
    y, acc, bad = oracle.moe_forward(**_hand_inputs(case), want_acc=True)
    yf = oracle.bf16_bits_to_float(y)[0]
    assert bad == 0
    if "y_all" in spec:
        assert np.all(yf == spec["y_all"][0])
    else:
        head = spec["y_head"]
        assert list(yf[:len(head)]) == head
        assert np.all(yf[len(head):] == spec["y_tail"][0])


# ---------------------------------------------- independent formulations
def _small_inputs(T, H, I, E, k, seed, mode=0):
    x, x_sf = synth.make_x(T, H, seed)
    w1, w1_sf = synth.make_w(E, 2 * I, H, 2, seed)
    w2, w2_sf = synth.make_w(E, H, I, 3, seed)
    idx, tw = synth.make_routing(T, E, k, mode, 0.0, seed)
    return dict(x=x, x_sf=x_sf, topk_idx=idx, topk_w=tw, w1=w1, w1_sf=w1_sf, w2=w2, w2_sf=w2_sf)


def test_dense_ffn_special_case():
    """E=1, k=1, weight 1: the layer is a dense two-layer FFN on every token."""
    d = _small_inputs(16, 256, 128, 1, 1, seed=3)
    d["topk_w"][:] = 1.0
    y, acc, _ = oracle.moe_forward(**d, want_acc=True)
    X = ind.dequant_x(d["x"], d["x_sf"])
    W1 = ind.dequant_w(d["w1"], d["w1_sf"])[0]
    W2 = ind.dequant_w(d["w2"], d["w2_sf"])[0]
    G = X @ W1.T
    a = (G[:, :128] / (1 + np.exp(-G[:, :128])) * G[:, 128:]).astype(np.float32)
    ad, _, _ = ind.requant(a)
    ref = ad @ W2.T  # weight 1: the accumulator is the FFN output itself
    np.testing.assert_allclose(acc, ref, rtol=1e-11, atol=1e-12 * np.abs(ref).max())


@pytest.mark.parametrize("T,E,k", [(4, 3, 2), (3, 2, 1), (4, 3, 3)])
def test_masked_all_experts_brute_force(T, E, k):
    d = _small_inputs(T, 128, 128, E, k, seed=T + E + k)
    y, acc, _ = oracle.moe_forward(**d, want_acc=True)
    ref = ind.moe_masked(**d)
    np.testing.assert_allclose(acc, ref, rtol=1e-11, atol=1e-12 * np.abs(ref).max())
    # y is the one BF16 rounding of that double sum (no per-slot rounding before it)
    assert np.array_equal(oracle.bf16_bits_to_float(y).astype(np.float64), ind.bf16_value(ref))


# ------------------------------------------------------------- invariants
@pytest.fixture(scope="module")
def tiny():
    return synth.make_inputs(synth.workload("tiny"))


@pytest.fixture(scope="module")
def tiny_y(tiny):
    return oracle.moe_forward(**tiny, want_acc=True)


def test_token_permutation_permutes_y(tiny, tiny_y):
    perm = np.random.default_rng(4).permutation(tiny["x"].shape[0])
    d = dict(tiny)
    for key in ("x", "x_sf", "topk_idx", "topk_w"):
        d[key] = np.ascontiguousarray(tiny[key][perm])
    y2, _, _ = oracle.moe_forward(**d)
    assert np.array_equal(y2, tiny_y[0][perm])


def test_slot_permutation_within_tolerance(tiny, tiny_y):
    d = dict(tiny)
    d["topk_idx"] = np.ascontiguousarray(tiny["topk_idx"][:, ::-1])
    d["topk_w"] = np.ascontiguousarray(tiny["topk_w"][:, ::-1])
    _, acc2, _ = oracle.moe_forward(**d, want_acc=True)
    np.testing.assert_allclose(acc2, tiny_y[1], rtol=1e-12, atol=1e-14)


def test_doubling_weights_doubles_y(tiny, tiny_y):
    d = dict(tiny)
    d["topk_w"] = tiny["topk_w"] * np.float32(2.0)
    y2, acc2, _ = oracle.moe_forward(**d, want_acc=True)
    assert np.array_equal(acc2, 2 * tiny_y[1])
    assert np.array_equal(oracle.bf16_bits_to_float(y2), 2 * oracle.bf16_bits_to_float(tiny_y[0]))


def test_poisoned_empty_experts_do_not_matter(tiny, tiny_y):
    d = dict(tiny)
    used = np.unique(tiny["topk_idx"])
    d["topk_idx"] = np.where(tiny["topk_idx"] == used[0], used[1], tiny["topk_idx"]).astype(np.int32)
    y_ref, _, _ = oracle.moe_forward(**d)
    empty = used[0]
    for key in ("w1", "w1_sf", "w2", "w2_sf"):
        d[key] = tiny[key].copy()
        d[key][empty] = 0xFF
    y2, _, _ = oracle.moe_forward(**d)
    assert np.array_equal(y2, y_ref)


def test_unused_slots_contribute_nothing(tiny, tiny_y):
    d = dict(tiny)
    idx = tiny["topk_idx"].copy()
    idx[:, 1] = -1
    d["topk_idx"] = idx
    y2, acc2, bad = oracle.moe_forward(**d, want_acc=True)
    d1 = dict(tiny)
    d1["topk_idx"] = np.ascontiguousarray(tiny["topk_idx"][:, :1])
    d1["topk_w"] = np.ascontiguousarray(tiny["topk_w"][:, :1])
    y1, acc1, _ = oracle.moe_forward(**d1, want_acc=True)
    assert bad == 0 and np.array_equal(acc2, acc1)


def test_token_subset_matches_full(tiny, tiny_y):
    toks = np.array([5, 0, 63, 17], np.int32)
    y2, _, _ = oracle.moe_forward(**tiny, tokens=toks)
    assert np.array_equal(y2, tiny_y[0][toks])
