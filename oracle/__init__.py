"""CPU oracle for the FP8 x FP4 MoE layer forward (test infrastructure).

This package is TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke``
and the CPU-baseline leg of ``bench.py`` may import it.  The product library
(``block_scaled_fp8_permute_b200``) never imports, links or calls it.

The arithmetic lives in ``moe_oracle.c`` (plain C, double precision, one
OpenMP loop over tokens).  This module compiles it with gcc into
``oracle/_build/liboracle.so`` and exposes thin numpy wrappers.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle C source into a shared library (gcc, -O2, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    c_u8p = ctypes.POINTER(ctypes.c_uint8)
    c_i32p = ctypes.POINTER(ctypes.c_int32)
    lib.orc_e2m1_value.restype = ctypes.c_double
    lib.orc_e2m1_value.argtypes = [ctypes.c_uint]
    lib.orc_e4m3_value.restype = ctypes.c_double
    lib.orc_e4m3_value.argtypes = [ctypes.c_uint]
    lib.orc_ue8m0_value.restype = ctypes.c_double
    lib.orc_ue8m0_value.argtypes = [ctypes.c_uint]
    lib.orc_e4m3_encode.restype = ctypes.c_uint
    lib.orc_e4m3_encode.argtypes = [ctypes.c_double]
    lib.orc_block_exponent.restype = ctypes.c_int
    lib.orc_block_exponent.argtypes = [ctypes.c_double, ctypes.c_double]
    lib.orc_silu.restype = ctypes.c_double
    lib.orc_silu.argtypes = [ctypes.c_double]
    lib.orc_bf16_rne.restype = ctypes.c_uint16
    lib.orc_bf16_rne.argtypes = [ctypes.c_double]
    lib.orc_requant_block.restype = None
    lib.orc_requant_block.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_int, c_u8p, c_u8p]
    lib.orc_plan.restype = ctypes.c_int
    lib.orc_plan.argtypes = [ctypes.c_int] * 4 + [c_i32p] * 6 + [ctypes.c_int]
    lib.orc_moe_forward.restype = ctypes.c_int
    lib.orc_moe_forward.argtypes = (
        [ctypes.c_int] * 5
        + [c_u8p, c_i32p, c_i32p, ctypes.POINTER(ctypes.c_float), c_u8p, c_u8p, c_u8p, c_u8p,
           c_i32p, ctypes.c_int, ctypes.POINTER(ctypes.c_uint16),
           ctypes.POINTER(ctypes.c_double), ctypes.c_int])
    lib.orc_gemm.restype = None
    lib.orc_gemm.argtypes = ([ctypes.c_int] * 4 + [c_u8p, c_i32p, c_i32p, c_u8p, c_u8p,
                                                   ctypes.POINTER(ctypes.c_uint16), ctypes.c_int])
    lib.orc_mqa_logits.restype = None
    lib.orc_mqa_logits.argtypes = ([ctypes.c_int] * 4 + [c_u8p, c_i32p, c_u8p, c_u8p,
                                                          ctypes.POINTER(ctypes.c_float), c_i32p,
                                                          c_i32p, ctypes.c_int,
                                                          ctypes.POINTER(ctypes.c_float),
                                                          ctypes.POINTER(ctypes.c_double),
                                                          ctypes.c_int])
    lib.orc_max_threads.restype = ctypes.c_int
    lib.orc_max_threads.argtypes = []
    _lib = lib
    return lib


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


# ---------------------------------------------------------------- codebooks
def e2m1_value(code: int) -> float:
    return _load().orc_e2m1_value(code)


def e4m3_value(code: int) -> float:
    return _load().orc_e4m3_value(code)


def ue8m0_value(code: int) -> float:
    return _load().orc_ue8m0_value(code)


def e4m3_encode(v: float) -> int:
    return _load().orc_e4m3_encode(float(v))


def block_exponent(amax: float, qmax: float) -> int:
    return _load().orc_block_exponent(float(amax), float(qmax))


def silu(z: float) -> float:
    return _load().orc_silu(float(z))


def bf16_rne(v: float) -> int:
    return _load().orc_bf16_rne(float(v))


def requant_rows(a: np.ndarray):
    """Requantise a float32 [rows, cols] array per 1x32 block along cols.

    Returns (codes u8 [rows, cols], scale bytes u8 [rows, cols/32])."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    rows, cols = a.shape
    assert cols % 32 == 0
    codes = np.zeros((rows, cols), np.uint8)
    sbytes = np.zeros((rows, cols // 32), np.uint8)
    lib = _load()
    for r in range(rows):
        for b in range(cols // 32):
            blk = np.ascontiguousarray(a[r, 32 * b:32 * b + 32])
            c = np.zeros(32, np.uint8)
            s = np.zeros(1, np.uint8)
            lib.orc_requant_block(_ptr(blk, ctypes.c_float), 32, _ptr(c, ctypes.c_uint8),
                                  _ptr(s, ctypes.c_uint8))
            codes[r, 32 * b:32 * b + 32] = c
            sbytes[r, b] = s[0]
    return codes, sbytes


# --------------------------------------------------------------------- plan
def plan(topk_idx: np.ndarray, E: int, bm: int):
    """Counting sort of assignments by expert, stable in t*k+s.

    Returns dict(counts, offs, poffs, row_of, src_of, P, bad)."""
    idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    T, k = idx.shape
    R = T * k
    counts = np.zeros(E, np.int32)
    offs = np.zeros(E + 1, np.int32)
    poffs = np.zeros(E + 1, np.int32)
    row_of = np.zeros(R, np.int32)
    p_cap = R + min(E, max(R, 1)) * bm + bm
    src_of = np.zeros(p_cap, np.int32)
    bad = _load().orc_plan(T, k, E, bm, _ptr(idx, ctypes.c_int32), _ptr(counts, ctypes.c_int32),
                           _ptr(offs, ctypes.c_int32), _ptr(poffs, ctypes.c_int32),
                           _ptr(row_of, ctypes.c_int32), _ptr(src_of, ctypes.c_int32), p_cap)
    P = int(poffs[E])
    return dict(counts=counts, offs=offs, poffs=poffs, row_of=row_of.reshape(T, k),
                src_of=src_of[:P].copy(), P=P, bad=bad)


# ------------------------------------------------------------------ forward
def moe_forward(x, x_sf, topk_idx, topk_w, w1, w1_sf, w2, w2_sf, tokens=None,
                want_acc=False, nthreads=0):
    """y (bf16 bits, uint16 [n, H]) for the listed tokens (all by default).

    Shapes (canonical layouts): x u8 [T,H]; x_sf i32 [T,H/128];
    topk_idx i32 [T,k]; topk_w f32 [T,k]; w1 u8 [E,2I,H/2]; w1_sf u8 [E,2I,H/32];
    w2 u8 [E,H,I/2]; w2_sf u8 [E,H,I/32].  Returns (y, acc or None, bad)."""
    T, H = x.shape
    E, twoI, _ = w1.shape
    I = twoI // 2
    k = topk_idx.shape[1]
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    n = tokens.shape[0]
    arrs = [np.ascontiguousarray(a) for a in (x, x_sf, topk_idx, topk_w, w1, w1_sf, w2, w2_sf)]
    x, x_sf, topk_idx, topk_w, w1, w1_sf, w2, w2_sf = arrs
    assert x.dtype == np.uint8 and x_sf.dtype == np.int32 and topk_idx.dtype == np.int32
    assert topk_w.dtype == np.float32 and w1.dtype == np.uint8 and w2.dtype == np.uint8
    y = np.zeros((n, H), np.uint16)
    acc = np.zeros((n, H), np.float64) if want_acc else None
    bad = _load().orc_moe_forward(
        T, H, I, E, k, _ptr(x, ctypes.c_uint8), _ptr(x_sf, ctypes.c_int32),
        _ptr(topk_idx, ctypes.c_int32), _ptr(topk_w, ctypes.c_float),
        _ptr(w1, ctypes.c_uint8), _ptr(w1_sf, ctypes.c_uint8), _ptr(w2, ctypes.c_uint8),
        _ptr(w2_sf, ctypes.c_uint8), _ptr(tokens, ctypes.c_int32), n,
        _ptr(y, ctypes.c_uint16),
        _ptr(acc, ctypes.c_double) if acc is not None else None, int(nthreads))
    return y, acc, bad


def gemm(a, a_sf, b, b_sf, masked_m=None, out=None, nthreads=0):
    """FP8 x FP4 GEMM, BF16 out (bits).  a u8 [G, M, K] (or [M, K]); a_sf i32
    [G, M, K/128]; b u8 [G, N, K/2] (or [N, K/2]); b_sf u8 [G, N, K/32];
    masked_m i32 [G] or None.  Rows at and beyond masked_m[g] keep the value
    they have in `out` (zeros when `out` is None)."""
    dense = a.ndim == 2
    a3 = np.ascontiguousarray(a if not dense else a[None], np.uint8)
    as3 = np.ascontiguousarray(a_sf if not dense else a_sf[None], np.int32)
    b3 = np.ascontiguousarray(b if b.ndim == 3 else b[None], np.uint8)
    bs3 = np.ascontiguousarray(b_sf if b_sf.ndim == 3 else b_sf[None], np.uint8)
    G, M, K = a3.shape
    N = b3.shape[1]
    d = np.zeros((G, M, N), np.uint16) if out is None else np.ascontiguousarray(
        out.reshape(G, M, N), np.uint16).copy()
    mm = None if masked_m is None else np.ascontiguousarray(masked_m, np.int32)
    _load().orc_gemm(G, M, N, K, _ptr(a3, ctypes.c_uint8), _ptr(as3, ctypes.c_int32),
                     _ptr(mm, ctypes.c_int32) if mm is not None else None,
                     _ptr(b3, ctypes.c_uint8), _ptr(bs3, ctypes.c_uint8),
                     _ptr(d, ctypes.c_uint16), int(nthreads))
    return d[0] if dense else d


def mqa_logits(q, q_sf, kv, kv_sf, weights, ks, ke, clean=True, want_mag=False, nthreads=0):
    """FP4-indexer logits, float32 [S, N] (entries outside [ks, ke) are -inf
    when clean, else NaN as 'not written').  q u8 [S, Hh, D]; q_sf i32
    [S, Hh, D/128]; kv u8 [N, D/2]; kv_sf u8 [N, D/32]; weights f32 [S, Hh];
    ks, ke i32 [S].  Returns (logits, mag or None)."""
    q = np.ascontiguousarray(q, np.uint8)
    S, Hh, D = q.shape
    N = kv.shape[0]
    arrs = [np.ascontiguousarray(a) for a in (q_sf, kv, kv_sf)]
    q_sf, kv, kv_sf = arrs
    w = np.ascontiguousarray(weights, np.float32)
    ks = np.ascontiguousarray(ks, np.int32)
    ke = np.ascontiguousarray(ke, np.int32)
    assert q_sf.dtype == np.int32 and kv.dtype == np.uint8 and kv_sf.dtype == np.uint8
    out = np.full((S, N), np.nan, np.float32)
    mag = np.zeros((S, N), np.float64) if want_mag else None
    _load().orc_mqa_logits(S, Hh, D, N, _ptr(q, ctypes.c_uint8), _ptr(q_sf, ctypes.c_int32),
                           _ptr(kv, ctypes.c_uint8), _ptr(kv_sf, ctypes.c_uint8),
                           _ptr(w, ctypes.c_float), _ptr(ks, ctypes.c_int32),
                           _ptr(ke, ctypes.c_int32), 1 if clean else 0,
                           _ptr(out, ctypes.c_float),
                           _ptr(mag, ctypes.c_double) if mag is not None else None, int(nthreads))
    return out, mag


def max_threads() -> int:
    return _load().orc_max_threads()


def bf16_bits_to_float(y: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 values."""
    return (y.astype(np.uint32) << 16).view(np.float32)
