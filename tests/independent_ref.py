"""A second, independently written formulation of the MoE layer in numpy.

Used only to pin the C oracle: it decodes the formats with vectorised bit
operations, requantises by nearest-value search over a sorted codebook, and
computes the layer as dense matrix products per expert with a mask over all
experts (no permutation, no plan).  It shares no code with the oracle or the
CUDA library.
"""
from __future__ import annotations

import numpy as np


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    c = codes.astype(np.int64) & 0xF
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, (e - 1).astype(np.int32)))
    return np.where(s == 1, -mag, mag)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    c = codes.astype(np.int64) & 0xFF
    s, e, m = (c >> 7) & 1, (c >> 3) & 0xF, c & 7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int32)))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def ue8m0_decode(b: np.ndarray) -> np.ndarray:
    b = b.astype(np.int64) & 0xFF
    return np.where(b == 255, np.nan, np.ldexp(1.0, (b - 127).astype(np.int32)))


_E4M3_MAG = e4m3_decode(np.arange(0x7F))          # codes 0x00..0x7E ascending


def e4m3_nearest(v: np.ndarray) -> np.ndarray:
    """Nearest E4M3 code, ties to the even code, saturating at 448."""
    a = np.abs(v)
    hi = np.clip(np.searchsorted(_E4M3_MAG, a, side="left"), 1, 0x7E)
    lo = hi - 1
    dl, dh = a - _E4M3_MAG[lo], _E4M3_MAG[hi] - a
    pick = np.where(dl < dh, lo, np.where(dh < dl, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a >= 448.0, 0x7E, pick)
    pick = np.where(a <= 0.0, 0, pick)
    return (pick | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)


def block_exponent(amax: np.ndarray, qmax: float) -> np.ndarray:
    """Smallest e with qmax * 2^e >= amax (0 for amax == 0), clamp +-127."""
    amax = np.asarray(amax, np.float64)
    _, ex = np.frexp(np.where(amax > 0, amax / qmax, 1.0))
    e = ex.astype(np.int64) - 1
    for _ in range(3):
        e = np.where(np.ldexp(qmax, e.astype(np.int32)) < amax, e + 1, e)
    for _ in range(3):
        e = np.where(np.ldexp(qmax, (e - 1).astype(np.int32)) >= amax, e - 1, e)
    e = np.where(amax > 0, e, 0)
    return np.clip(e, -127, 127)


def requant(a32: np.ndarray):
    """a32 float32 [rows, I] -> (decoded values float64, codes, scale bytes)."""
    rows, cols = a32.shape
    blk = a32.astype(np.float64).reshape(rows, cols // 32, 32)
    e = block_exponent(np.abs(blk).max(axis=2), 448.0)
    q = e4m3_nearest(np.ldexp(blk, -e[:, :, None].astype(np.int32)))
    dec = e4m3_decode(q) * np.ldexp(1.0, e[:, :, None].astype(np.int32))
    return dec.reshape(rows, cols), q.reshape(rows, cols), (e + 127).astype(np.uint8)


def dequant_x(x: np.ndarray, x_sf: np.ndarray) -> np.ndarray:
    T, H = x.shape
    sbytes = x_sf.view(np.uint8).reshape(T, H // 32)        # little-endian bytes in block order
    return e4m3_decode(x) * np.repeat(ue8m0_decode(sbytes), 32, axis=1)


def dequant_w(w: np.ndarray, w_sf: np.ndarray) -> np.ndarray:
    E, N, Kh = w.shape
    lo, hi = w & 0xF, w >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(E, N, 2 * Kh)
    return e2m1_decode(codes) * np.repeat(ue8m0_decode(w_sf), 32, axis=2)


def bf16_round(v: np.ndarray) -> np.ndarray:
    """Round float64 -> bf16 (RNE) through torch's float32 -> bf16 cast.

    Valid when the float64 values are exactly representable in float32 or
    when the caller accepts double rounding (used only for exact cases)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_value(v: np.ndarray) -> np.ndarray:
    """float64 -> nearest bf16 value (ties to even), returned as float64.

    bf16 keeps 8 significant bits: with |v| = m * 2^e, m in [0.5, 1), the
    grid step is 2^(e-8); below 2^-126 the step stays 2^-133 (subnormals)."""
    v = np.asarray(v, np.float64)
    _, e = np.frexp(np.abs(v))
    e = np.maximum(e, -125)
    q = np.ldexp(np.rint(np.ldexp(np.abs(v), 8 - e)), e - 8)
    return np.copysign(q, v)


def moe_masked(x, x_sf, topk_idx, topk_w, w1, w1_sf, w2, w2_sf):
    """Masked all-experts formulation:
    acc[t] = sum_e sum_s [idx[t,s]==e] w[t,s] FFN_e(x_t).

    Returns the float64 accumulator [T, H]."""
    T, H = x.shape
    E = w1.shape[0]
    I = w1.shape[1] // 2
    X = dequant_x(x, x_sf)
    W1 = dequant_w(w1, w1_sf)
    W2 = dequant_w(w2, w2_sf)
    acc = np.zeros((T, H))
    for e in range(E):
        G = X @ W1[e].T                                   # [T, 2I]
        gate, up = G[:, :I], G[:, I:]
        a = (gate / (1.0 + np.exp(-gate)) * up).astype(np.float32)
        ad, _, _ = requant(a)
        O = ad @ W2[e].T                                  # [T, H]
        for s in range(topk_idx.shape[1]):
            sel = (topk_idx[:, s] == e).astype(np.float64) * topk_w[:, s].astype(np.float64)
            acc += sel[:, None] * O
    return acc


def mqa_logits(q, q_sf, kv, kv_sf, weights, ks, ke):
    """FP4-indexer logits written independently: decode q and k to float64,
    per-head dot products as one matmul, ReLU, weighted head sum; entries
    outside [ks, ke) are -inf.  Returns float64 [S, N]."""
    S, Hh, D = q.shape
    N = kv.shape[0]
    Q = dequant_x(q.reshape(S * Hh, D), q_sf.reshape(S * Hh, D // 128)).reshape(S, Hh, D)
    K = dequant_w(kv[None], kv_sf[None])[0]                       # [N, D]
    dots = np.einsum("shd,nd->shn", Q, K)                        # [S, Hh, N]
    out = np.einsum("sh,shn->sn", weights.astype(np.float64), np.maximum(dots, 0.0))
    j = np.arange(N)[None, :]
    valid = (j >= np.maximum(ks, 0)[:, None]) & (j < np.minimum(ke, N)[:, None])
    return np.where(valid, out, -np.inf)
