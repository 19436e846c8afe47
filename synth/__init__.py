"""Seeded synthetic workloads for the FP8 x FP4 MoE layer forward.

Input preparation only (no layer arithmetic): both the CUDA library's tests
and bench, and the CPU oracle, take their inputs from here.  The C source
``synth.c`` draws counter-based normals and casts them to the formats the
layer consumes; this module compiles it and names the workloads.

Workloads (seed 0 everywhere):
  tiny     T=64,   H=256,  E=8,   k=2, I=512,  softmax over the chosen 2
  mid      T=4096, H=2048, E=32,  k=4, I=1024, softmax over the chosen 4
  usage    T=8192, H=7168, E=8,   k=2, I=9216, softmax over the chosen 2
           (the shape of the Mega MoE usage example: 18432 = gate + up)
  skewed   T=4096, H=7168, E=256, k=8, I=2048, logits + Zipf(1.1) bias,
           sigmoid of the chosen 8, renormalised
  decode   T=128 (also 16, 32, 64), H=7168, E=256, k=8, I=2048, sigmoid of
           the chosen 8, renormalised, no bias
Weights ~ N(0, 1/K) (std 1/sqrt(K), K = H for W1 and I for W2); x ~ N(0, 1).
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libsynth.so")
_lib = None


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    mode: int          # 0 softmax over chosen, 1 sigmoid of chosen / sum
    zipf_s: float      # > 0: add the Zipf per-expert bias to the logits
    seed: int = 0

    @property
    def R(self) -> int:
        return self.T * self.k

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs: 2*R*H*2I (linear1) + 2*R*I*H (linear2)."""
        return 6.0 * self.T * self.k * self.H * self.I

    def with_tokens(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T, name=f"{self.name.split('@')[0]}@T{T}")


WORKLOADS = {
    "tiny": Workload("tiny", 64, 256, 8, 2, 512, 0, 0.0),
    "mid": Workload("mid", 4096, 2048, 32, 4, 1024, 0, 0.0),
    "usage": Workload("usage", 8192, 7168, 8, 2, 9216, 0, 0.0),
    "skewed": Workload("skewed", 4096, 7168, 256, 8, 2048, 1, 1.1),
    "decode": Workload("decode", 128, 7168, 256, 8, 2048, 1, 0.0),
    # a profiling-sized decode layer: the decode shape with 64 experts (1.4 GB of
    # FP4 weights, still far above L2), small enough for a multi-pass ncu capture
    "decode-e64": Workload("decode-e64", 128, 7168, 64, 8, 2048, 1, 0.0),
}


def build(force: bool = False) -> str:
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                    "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u8p, i32p = ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(ctypes.c_int32)
        lib.synth_x.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_uint64, u8p, i32p]
        lib.synth_w.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                ctypes.c_uint64, ctypes.c_double, u8p, u8p]
        lib.synth_routing.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                      ctypes.c_int, ctypes.c_double, i32p,
                                      ctypes.POINTER(ctypes.c_float)]
        _lib = lib
    return _lib


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def make_x(T: int, H: int, seed: int = 0):
    x = np.empty((T, H), np.uint8)
    x_sf = np.zeros((T, H // 128), np.int32)
    _load().synth_x(T, H, seed, _p(x, ctypes.c_uint8), _p(x_sf, ctypes.c_int32))
    return x, x_sf


def make_w(E: int, N: int, K: int, stream: int, seed: int = 0, std: float | None = None):
    if std is None:
        std = 1.0 / math.sqrt(K)
    w = np.empty((E, N, K // 2), np.uint8)
    w_sf = np.empty((E, N, K // 32), np.uint8)
    _load().synth_w(E, N, K, seed, stream, std, _p(w, ctypes.c_uint8), _p(w_sf, ctypes.c_uint8))
    return w, w_sf


def make_routing(T: int, E: int, k: int, mode: int, zipf_s: float, seed: int = 0):
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    _load().synth_routing(T, E, k, seed, mode, zipf_s, _p(idx, ctypes.c_int32),
                          _p(w, ctypes.c_float))
    return idx, w


def make_weights(wl: Workload):
    w1, w1_sf = make_w(wl.E, 2 * wl.I, wl.H, stream=2, seed=wl.seed)
    w2, w2_sf = make_w(wl.E, wl.H, wl.I, stream=3, seed=wl.seed)
    return w1, w1_sf, w2, w2_sf


def make_activations(wl: Workload):
    x, x_sf = make_x(wl.T, wl.H, seed=wl.seed)
    idx, w = make_routing(wl.T, wl.E, wl.k, wl.mode, wl.zipf_s, seed=wl.seed)
    return x, x_sf, idx, w


def make_inputs(wl: Workload) -> dict:
    x, x_sf, idx, tw = make_activations(wl)
    w1, w1_sf, w2, w2_sf = make_weights(wl)
    return dict(x=x, x_sf=x_sf, topk_idx=idx, topk_w=tw, w1=w1, w1_sf=w1_sf, w2=w2, w2_sf=w2_sf)


def workload(name: str) -> Workload:
    """'mid', 'decode', or 'decode@T32' style names."""
    if "@T" in name:
        base, t = name.split("@T")
        return WORKLOADS[base].with_tokens(int(t))
    return WORKLOADS[name]


# ------------------------------------------------------------ FP4 indexer
@dataclasses.dataclass(frozen=True)
class IndexerWorkload:
    """MQA-logit workload of the FP4 indexer: S query tokens with Hh heads of
    dimension D against N keys; query i sees keys [0, N - S + i + 1) (the
    keys already cached plus the new tokens up to itself)."""
    name: str
    S: int
    Hh: int
    D: int
    N: int
    seed: int = 0

    @property
    def pairs(self) -> int:
        """(query, key) pairs inside the ranges."""
        return sum(self.N - self.S + i + 1 for i in range(self.S))

    @property
    def flops(self) -> float:
        """2 * Hh * D per scored pair (the dot products; the weighted ReLU sum is not counted)."""
        return 2.0 * self.Hh * self.D * self.pairs


INDEXER_WORKLOADS = {
    # prefill: 4096 new tokens over an 8192-token context, 64 index heads of dimension 128
    "indexer": IndexerWorkload("indexer", 4096, 64, 128, 8192),
    # decode with 4 multi-token-prediction tokens over a 65536-token context
    "indexer-decode": IndexerWorkload("indexer-decode", 4, 64, 128, 65536),
}


def make_indexer(S: int, Hh: int, D: int, N: int, seed: int = 0):
    """q u8 [S, Hh, D] E4M3 (+ q_sf i32 [S, Hh, D/128]) from the activation
    generator, kv u8 [N, D/2] E2M1 (+ kv_sf u8 [N, D/32]) from the weight
    generator (stream 6, std 1), weights f32 [S, Hh] ~ N(0, 1/Hh) and the
    prefix ranges ks = 0, ke = N - S + i + 1 (clamped to [0, N])."""
    q, q_sf = make_x(S * Hh, D, seed)
    kv, kv_sf = make_w(1, N, D, 6, seed, std=1.0)
    rng = np.random.default_rng(seed + 1000)
    w = (rng.standard_normal((S, Hh)) / math.sqrt(Hh)).astype(np.float32)
    ke = np.clip(N - S + 1 + np.arange(S), 0, N).astype(np.int32)
    ks = np.zeros(S, np.int32)
    return dict(q=q.reshape(S, Hh, D), q_sf=q_sf.reshape(S, Hh, D // 128), kv=kv[0],
                kv_sf=kv_sf[0], weights=w, ks=ks, ke=ke)
