"""Pins for the oracle's FP4-indexer logits (fp8_fp4_mqa_logits reading:
"DeepSeek DeepGEMM 2026年4月重磅更新" sections 5.1-5.2).

Pinned by hand-worked closed forms (tests/golden/indexer_hand.txt), an
independent numpy formulation (tests/independent_ref.py: vectorised decodes,
one einsum per head), the key-range contract (-inf outside [ks, ke), nothing
written without cleaning) and invariants (head permutation, weight scaling,
all-negative dots).
"""
import os

import numpy as np
import pytest

import oracle
import synth
from tests import independent_ref as ind


def _hand_inputs():
    S, Hh, D, N = 1, 2, 128, 3
    q = np.empty((S, Hh, D), np.uint8)
    q[0, 0] = 0x30
    q[0, 1] = 0xB8
    q_sf = np.full((S, Hh, 1), 0x7F7F7F7F, np.int32)
    codes = np.empty((N, D), np.uint8)
    codes[0], codes[1], codes[2] = 0x2, 0x1, 0xA
    kv = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    kv_sf = np.full((N, D // 32), 127, np.uint8)
    w = np.array([[2.0, 3.0]], np.float32)
    return q, q_sf, kv, kv_sf, w


def _read_cases(golden_dir):
    out = {}
    with open(os.path.join(golden_dir, "indexer_hand.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                p = line.split()
                out[p[0]] = (int(p[1]), int(p[2]), [float(v) for v in p[3:]])
    return out


@pytest.mark.parametrize("case", ["caseA", "caseB", "caseC"])
def test_hand_worked(golden_dir, case):
    ks, ke, want = _read_cases(golden_dir)[case]
    q, q_sf, kv, kv_sf, w = _hand_inputs()
    got, _ = oracle.mqa_logits(q, q_sf, kv, kv_sf, w, np.array([ks], np.int32),
                               np.array([ke], np.int32))
    assert list(got[0]) == want


def _inputs(S, Hh, D, N, seed):
    q, q_sf = synth.make_x(S * Hh, D, seed)
    kv, kv_sf = synth.make_w(1, N, D, 5, seed)
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((S, Hh)).astype(np.float32)
    ks = rng.integers(-2, N // 2, S).astype(np.int32)
    ke = (ks + rng.integers(0, N + 3, S)).astype(np.int32)
    return dict(q=q.reshape(S, Hh, D), q_sf=q_sf.reshape(S, Hh, D // 128), kv=kv[0],
                kv_sf=kv_sf[0], weights=w, ks=ks, ke=ke)


@pytest.mark.parametrize("S,Hh,D,N,seed", [(5, 3, 128, 40, 1), (3, 4, 256, 17, 2),
                                           (7, 1, 128, 9, 3)])
def test_matches_independent_formulation(S, Hh, D, N, seed):
    d = _inputs(S, Hh, D, N, seed)
    got, _ = oracle.mqa_logits(**d)
    ref = ind.mqa_logits(**d)
    assert np.array_equal(np.isinf(got), np.isinf(ref))
    fin = np.isfinite(ref)
    np.testing.assert_allclose(got[fin], ref[fin].astype(np.float32), rtol=1e-6, atol=1e-6)


def test_unclean_rows_are_not_written():
    d = _inputs(4, 2, 128, 20, 4)
    got, _ = oracle.mqa_logits(**d, clean=False)
    ref = ind.mqa_logits(**d)
    assert np.array_equal(np.isnan(got), np.isinf(ref))      # sentinel kept outside the range


def test_closed_form_all_ones():
    """q = 1, k = 1: every dot is D, so logit = D * sum_h w_h (all dots positive)."""
    S, Hh, D, N = 2, 4, 256, 5
    q = np.full((S, Hh, D), 0x38, np.uint8)
    q_sf = np.full((S, Hh, D // 128), 0x7F7F7F7F, np.int32)
    kv = np.full((N, D // 2), 0x22, np.uint8)
    kv_sf = np.full((N, D // 32), 127, np.uint8)
    w = np.array([[1.0, -2.0, 0.5, 4.0], [0.25, 0.25, 0.25, 0.25]], np.float32)
    got, _ = oracle.mqa_logits(q, q_sf, kv, kv_sf, w, np.zeros(S, np.int32),
                               np.full(S, N, np.int32))
    np.testing.assert_array_equal(got, np.repeat((D * w.sum(axis=1))[:, None], N, axis=1))


def test_negative_dots_vanish():
    d = _inputs(3, 2, 128, 10, 5)
    d2 = dict(d)
    d2["q"] = d["q"] ^ 0x80                              # flip every sign of q
    a, _ = oracle.mqa_logits(**d)
    b, _ = oracle.mqa_logits(**d2)
    ref_pos = ind.mqa_logits(**d)
    ref_neg = ind.mqa_logits(**d2)
    # ReLU(s) + ReLU(-s) = |s|: the two runs add up to the weighted sum of |dots|
    fin = np.isfinite(a)
    Q = ind.dequant_x(d["q"].reshape(-1, 128), d["q_sf"].reshape(-1, 1)).reshape(3, 2, 128)
    K = ind.dequant_w(d["kv"][None], d["kv_sf"][None])[0]
    absdot = np.einsum("sh,shn->sn", d["weights"].astype(np.float64),
                       np.abs(np.einsum("shd,nd->shn", Q, K)))
    np.testing.assert_allclose((a.astype(np.float64) + b)[fin], absdot[fin], rtol=1e-6, atol=1e-6)
    assert np.array_equal(np.isinf(ref_pos), np.isinf(ref_neg))


def test_head_permutation_and_weight_scaling():
    d = _inputs(4, 5, 128, 12, 6)
    base, _ = oracle.mqa_logits(**d)
    perm = np.random.default_rng(0).permutation(5)
    d2 = dict(d, q=np.ascontiguousarray(d["q"][:, perm]), q_sf=np.ascontiguousarray(d["q_sf"][:, perm]),
              weights=np.ascontiguousarray(d["weights"][:, perm]))
    p, _ = oracle.mqa_logits(**d2)
    fin = np.isfinite(base)
    np.testing.assert_allclose(p[fin], base[fin], rtol=1e-6, atol=1e-6)
    d3 = dict(d, weights=d["weights"] * np.float32(2.0))
    s, _ = oracle.mqa_logits(**d3)
    np.testing.assert_array_equal(s[fin], 2 * base[fin])
