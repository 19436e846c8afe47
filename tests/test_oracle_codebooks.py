"""Pins for the oracle's codebooks, encoder, scale rule, SwiGLU and bf16 rounding.

Each check compares the oracle with something other than itself: values the
formats' bit definitions fix (tests/golden/codebooks.txt, cited there),
exhaustive round trips, a brute-force nearest-code search, exact scale
boundaries, long-double arithmetic and torch's bf16 cast.
"""
import math
import os

import numpy as np
import pytest

import oracle


def _golden(golden_dir, name):
    rows = []
    with open(os.path.join(golden_dir, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(line.split())
    return rows


def _same(a, b):
    if math.isnan(b):
        return math.isnan(a)
    return a == b and math.copysign(1, a) == math.copysign(1, b)


def test_golden_codebook_values(golden_dir):
    fn = {"e2m1": oracle.e2m1_value, "e4m3": oracle.e4m3_value, "ue8m0": oracle.ue8m0_value}
    rows = _golden(golden_dir, "codebooks.txt")
    assert len(rows) >= 25
    for kind, code, val in rows:
        got = fn[kind](int(code, 0))
        assert _same(got, float(val)), (kind, code, val, got)


def test_e2m1_all_codes():
    vals = [oracle.e2m1_value(c) for c in range(16)]
    pos = vals[:8]
    assert pos == sorted(pos) and len(set(pos)) == 8
    for c in range(8):
        assert _same(vals[c + 8], -pos[c])


def test_e4m3_structure():
    vals = [oracle.e4m3_value(c) for c in range(256)]
    pos = vals[:0x7F]
    assert all(a < b for a, b in zip(pos, pos[1:]))            # strictly increasing
    assert pos[-1] == 448.0 and pos[1] == 2.0 ** -9
    assert math.isnan(vals[0x7F]) and math.isnan(vals[0xFF])
    for c in range(0x7F):
        assert _same(vals[c | 0x80], -pos[c])
    # 8 values per binade above the subnormals, subnormals evenly spaced by 2^-9
    for c in range(1, 8):
        assert pos[c] == c * 2.0 ** -9
    for e in range(1, 16):
        binade = [v for v in pos if 2.0 ** (e - 7) <= v < 2.0 ** (e - 6)]
        assert len(binade) == (8 if e < 15 else 7)


def test_ue8m0_all_codes():
    for b in range(255):
        assert oracle.ue8m0_value(b) == 2.0 ** (b - 127)
    assert math.isnan(oracle.ue8m0_value(255))


def test_e4m3_encode_roundtrip_all_finite_codes():
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        assert oracle.e4m3_encode(oracle.e4m3_value(c)) == c


def _brute_e4m3(v):
    """Nearest finite E4M3 by scanning every code; ties to the even code;
    saturating beyond 448."""
    best, bestd = None, None
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        cv = oracle.e4m3_value(c)
        if math.copysign(1, cv) != math.copysign(1, v):
            continue
        d = abs(cv - v)
        if bestd is None or d < bestd or (d == bestd and c % 2 == 0 and best % 2 == 1):
            best, bestd = c, d
    return best


def test_e4m3_encode_matches_brute_force():
    rng = np.random.default_rng(0)
    pos = [oracle.e4m3_value(c) for c in range(0x7F)]
    mids = [(a + b) / 2 for a, b in zip(pos, pos[1:])]
    grid = list(rng.uniform(-460, 460, 3000)) + list(rng.standard_normal(2000) * 0.05)
    grid += mids + [-m for m in mids] + [m * (1 + 1e-12) for m in mids] + [m * (1 - 1e-12) for m in mids]
    grid += [448.0, 449.0, 463.99, 464.0, 1e6, -1e6, 0.0, -0.0, 2.0 ** -10, 2.0 ** -11]
    for v in grid:
        want = _brute_e4m3(v) if abs(v) <= 448 else (0x7E | (0x80 if v < 0 else 0))
        assert oracle.e4m3_encode(v) == want, v


@pytest.mark.parametrize("qmax", [448.0, 6.0])
def test_block_exponent_boundaries(qmax):
    for e in range(-127, 128):
        edge = math.ldexp(qmax, e)
        assert oracle.block_exponent(edge, qmax) == e
        up = math.nextafter(edge, math.inf)
        if e < 127:
            assert oracle.block_exponent(up, qmax) == e + 1
        dn = math.nextafter(edge, 0.0)
        if e > -127:
            assert oracle.block_exponent(dn, qmax) == e
    assert oracle.block_exponent(0.0, qmax) == 0
    assert oracle.block_exponent(1e-300, qmax) == -127


def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    # sigmoid(ln 3) = 3/4
    assert abs(oracle.silu(math.log(3.0)) - 0.75 * math.log(3.0)) < 1e-15
    assert abs(oracle.silu(60.0) - 60.0) < 1e-20 * 60 + 1e-12
    assert oracle.silu(-50.0) < 0 and abs(oracle.silu(-50.0)) < 1e-19
    # against long-double arithmetic
    for z in np.linspace(-30, 30, 601):
        zl = np.longdouble(z)
        ref = zl / (np.longdouble(1) + np.exp(-zl))
        got = oracle.silu(float(z))
        assert abs(np.longdouble(got) - ref) <= 2 * np.spacing(abs(float(ref))) + 1e-300


def test_bf16_matches_torch_cast():
    import torch
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(4000).astype(np.float32),
                        (rng.standard_normal(1000) * 1e-30).astype(np.float32),
                        (rng.standard_normal(1000) * 1e30).astype(np.float32)])
    # exact ties: bf16 value + half an ulp
    ties = (np.arange(1, 200, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    v = np.concatenate([v, ties, -ties])
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_rne(float(a)) for a in v], np.uint16)
    assert np.array_equal(got, want)


def test_bf16_of_doubles_matches_independent_rounding():
    """Doubles that are not float32 values (the linear2 products the oracle
    rounds): the oracle's rounding against the numpy formulation in
    independent_ref, including exact ties and values a hair off a tie."""
    import independent_ref as ind
    rng = np.random.default_rng(7)
    v = rng.standard_normal(3000) * np.exp2(rng.integers(-40, 40, 3000))
    base = np.ldexp(rng.integers(128, 256, 500).astype(np.float64), rng.integers(-20, 20, 500))
    ulp = np.ldexp(1.0, np.frexp(base)[1] - 8)
    ties = base + 0.5 * ulp
    v = np.concatenate([v, ties, -ties, ties + ulp * 1e-9, ties - ulp * 1e-9])
    got = np.array([oracle.bf16_rne(float(a)) for a in v], np.uint16)
    want = ind.bf16_value(v)
    got_v = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(got_v, want)
    # exact ties go to the even neighbour: the significand's low bit is clear
    assert ((got[3000:3500] & 1) == 0).all()


def test_requant_block_matches_independent_formulation():
    from tests.independent_ref import requant
    rng = np.random.default_rng(2)
    a = (rng.standard_normal((64, 128)) * np.exp(rng.uniform(-8, 8, (64, 1)))).astype(np.float32)
    a[3, :32] = 0.0                                       # an all-zero block
    a[5, 32:64] = 448.0 * 2.0 ** 3                        # amax exactly on a boundary
    codes, sb = oracle.requant_rows(a)
    _, q2, e2 = requant(a)
    assert np.array_equal(codes, q2)
    assert np.array_equal(sb, e2)
    assert sb[3, 0] == 127 and np.all(codes[3, :32] == 0)
    assert sb[5, 1] == 127 + 3 and np.all(codes[5, 32:64] == 0x7E)
