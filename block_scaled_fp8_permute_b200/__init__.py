"""Python binding of libmoe, the B200 (sm_100a) FP8 x FP4 MoE layer forward.

Argument marshalling only: every step of the forward runs in the CUDA
kernels of ``libmoe.so`` (built in-tree by ``build.py``).  PyTorch supplies
device memory and streams.  The functions mirror the C ABI in
``include/moe.h`` name for name; each raises ``MoeError`` on a non-OK status.
There is no fallback: importing this package fails loudly when the library
has not been built.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libmoe.so not found at {LIB_PATH}; build it with "
        "`python block_scaled_fp8_permute_b200/build.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
                3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT",
                6: "MOE_ERR_BAD_EXPERT_ID"}


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


class MoeShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("H", ctypes.c_int), ("I", ctypes.c_int),
                ("E", ctypes.c_int), ("topk", ctypes.c_int)]

    def __repr__(self):
        return f"MoeShape(T={self.T}, H={self.H}, I={self.I}, E={self.E}, topk={self.topk})"


_vp, _sz, _i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
_shp = ctypes.POINTER(MoeShape)
_SIGS = {
    "moe_status_string": (ctypes.c_char_p, [_i]),
    "moe_block_m": (_i, []),
    "moe_set_num_sms": (None, [_i]),
    "moe_set_pdl": (None, [_i]),
    "moe_set_gemm_variant": (None, [_i]),
    "moe_set_swap_max": (None, [_i]),
    "moe_set_narrow_tiles": (None, [_i]),
    "moe_transformed_bytes": (_sz, [_shp, _i, ctypes.POINTER(_sz)]),
    "moe_transform_weights": (_i, [_shp] + [_vp] * 8 + [_vp]),
    "moe_workspace_bytes": (_sz, [_shp]),
    "moe_plan": (_i, [_shp, _vp, _vp, _sz, _vp]),
    "moe_forward": (_i, [_shp] + [_vp] * 9 + [_vp, _sz, _vp]),
    "moe_workspace_bytes_host": (_sz, [_shp]),
    "moe_forward_host": (_i, [_shp] + [_vp] * 9 + [_vp, _sz, _vp]),
    "moe_workspace_bytes_host_pipelined": (_sz, [_shp]),
    "moe_forward_host_pipelined": (_i, [_shp, _i] + [ctypes.POINTER(_vp)] * 4 + [_vp] * 4
                                   + [ctypes.POINTER(_vp), _vp, _sz, _vp]),
    "moe_get_device_status": (_i, [_vp, _vp]),
    "moe_get_timeout_site": (_i, [_vp, _vp]),
    "moe_debug_set_fault": (None, [_i, ctypes.c_ulonglong]),
    "moe_plan_max_rows": (_i, [_shp]),
    "moe_plan_export": (_i, [_shp, _vp] + [_vp] * 6 + [_vp]),
    "moe_debug_requant": (_i, [_vp, _i, _i, _vp, _vp, _vp]),
    "moe_set_timing_events": (None, [ctypes.POINTER(_vp), _i]),
    "moe_forward_noalloc": (_i, [_shp] + [_vp] * 9 + [_vp]),
    "moe_gemm_b_bytes": (_sz, [_i, _i, _i, ctypes.POINTER(_sz)]),
    "moe_gemm_transform_b": (_i, [_i, _i, _i] + [_vp] * 4 + [_vp]),
    "moe_gemm_workspace_bytes": (_sz, [_i, _i, _i, _i]),
    "moe_gemm_fp8_fp4": (_i, [_i, _i, _i] + [_vp] * 6 + [_sz, _vp]),
    "moe_gemm_fp8_fp4_masked": (_i, [_i, _i, _i, _i] + [_vp] * 7 + [_sz, _vp]),
    "moe_mqa_logits_workspace_bytes": (_sz, [_i, _i, _i, _i]),
    "moe_fp8_fp4_mqa_logits": (_i, [_i, _i, _i, _i] + [_vp] * 7 + [_i, _vp, _vp, _sz, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def lib():
    """The raw ctypes handle of libmoe.so."""
    return _lib


def _check(fn: str, st: int):
    if st != MOE_OK:
        raise MoeError(fn, st)


def _ptr(t):
    """Device (or host) address of a tensor / numpy array / int / None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    return t.ctypes.data  # numpy


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def shape(T, H, I, E, topk) -> MoeShape:
    return MoeShape(T, H, I, E, topk)


# ------------------------------------------------------------------ C ABI
def moe_status_string(status: int) -> str:
    return _lib.moe_status_string(status).decode()


def moe_block_m() -> int:
    return _lib.moe_block_m()


def moe_set_num_sms(n: int) -> None:
    _lib.moe_set_num_sms(n)


def moe_set_pdl(enable: bool) -> None:
    _lib.moe_set_pdl(1 if enable else 0)


def moe_set_gemm_variant(variant: int) -> None:
    _lib.moe_set_gemm_variant(variant)


def moe_set_swap_max(rows: int) -> None:
    _lib.moe_set_swap_max(rows)


def moe_set_narrow_tiles(mode: int) -> None:
    _lib.moe_set_narrow_tiles(mode)


def moe_transformed_bytes(shp: MoeShape, which: int):
    sf = _sz(0)
    n = _lib.moe_transformed_bytes(ctypes.byref(shp), which, ctypes.byref(sf))
    return n, sf.value


def moe_transform_weights(shp, w1, w1_sf, w2, w2_sf, w1_t, w1_sf_t, w2_t, w2_sf_t, stream=None):
    _check("moe_transform_weights", _lib.moe_transform_weights(
        ctypes.byref(shp), _ptr(w1), _ptr(w1_sf), _ptr(w2), _ptr(w2_sf), _ptr(w1_t),
        _ptr(w1_sf_t), _ptr(w2_t), _ptr(w2_sf_t), _stream(stream)))


def moe_workspace_bytes(shp: MoeShape) -> int:
    return _lib.moe_workspace_bytes(ctypes.byref(shp))


def moe_workspace_bytes_host(shp: MoeShape) -> int:
    return _lib.moe_workspace_bytes_host(ctypes.byref(shp))


def moe_plan(shp, topk_idx, workspace, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check("moe_plan", _lib.moe_plan(ctypes.byref(shp), _ptr(topk_idx), _ptr(workspace),
                                     ws_bytes, _stream(stream)))


def moe_forward(shp, x, x_sf, topk_idx, topk_w, w1_t, w1_sf_t, w2_t, w2_sf_t, y, workspace,
                ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check("moe_forward", _lib.moe_forward(
        ctypes.byref(shp), _ptr(x), _ptr(x_sf), _ptr(topk_idx), _ptr(topk_w), _ptr(w1_t),
        _ptr(w1_sf_t), _ptr(w2_t), _ptr(w2_sf_t), _ptr(y), _ptr(workspace), ws_bytes,
        _stream(stream)))


def moe_forward_host(shp, x, x_sf, topk_idx, topk_w, w1_t, w1_sf_t, w2_t, w2_sf_t, y, workspace,
                     ws_bytes=None, stream=None):
    """x, x_sf, topk_idx, topk_w and y are HOST buffers (pinned torch tensors
    or numpy arrays); weights and workspace live on the device."""
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check("moe_forward_host", _lib.moe_forward_host(
        ctypes.byref(shp), _ptr(x), _ptr(x_sf), _ptr(topk_idx), _ptr(topk_w), _ptr(w1_t),
        _ptr(w1_sf_t), _ptr(w2_t), _ptr(w2_sf_t), _ptr(y), _ptr(workspace), ws_bytes,
        _stream(stream)))


def moe_workspace_bytes_host_pipelined(shp: MoeShape) -> int:
    return _lib.moe_workspace_bytes_host_pipelined(ctypes.byref(shp))


def moe_forward_host_pipelined(shp, xs, x_sfs, topk_idxs, topk_ws, w1_t, w1_sf_t, w2_t, w2_sf_t,
                               ys, workspace, ws_bytes=None, stream=None):
    """len(xs) successive host-buffer forwards: xs, x_sfs, topk_idxs, topk_ws
    and ys are equal-length lists of HOST buffers (pinned torch tensors or
    numpy arrays), batch i reading the i-th of each and writing ys[i]."""
    n = len(xs)
    if not (len(x_sfs) == len(topk_idxs) == len(topk_ws) == len(ys) == n):
        raise ValueError("moe_forward_host_pipelined: the buffer lists differ in length")
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()

    def arr(bufs):
        return (_vp * max(n, 1))(*[_ptr(b) for b in bufs])

    _check("moe_forward_host_pipelined", _lib.moe_forward_host_pipelined(
        ctypes.byref(shp), n, arr(xs), arr(x_sfs), arr(topk_idxs), arr(topk_ws), _ptr(w1_t),
        _ptr(w1_sf_t), _ptr(w2_t), _ptr(w2_sf_t), arr(ys), _ptr(workspace), ws_bytes,
        _stream(stream)))


def moe_forward_noalloc(shp, x, x_sf, topk_idx, topk_w, w1_t, w1_sf_t, w2_t, w2_sf_t, y,
                        stream=None):
    """moe_plan + moe_forward on the library's own fixed 32 MiB workspace
    (for callers that cannot allocate device memory)."""
    _check("moe_forward_noalloc", _lib.moe_forward_noalloc(
        ctypes.byref(shp), _ptr(x), _ptr(x_sf), _ptr(topk_idx), _ptr(topk_w), _ptr(w1_t),
        _ptr(w1_sf_t), _ptr(w2_t), _ptr(w2_sf_t), _ptr(y), _stream(stream)))


def moe_get_device_status(workspace, stream=None) -> int:
    return _lib.moe_get_device_status(_ptr(workspace), _stream(stream))


def moe_get_timeout_site(workspace, stream=None) -> int:
    return _lib.moe_get_timeout_site(_ptr(workspace), _stream(stream))


def moe_debug_set_fault(skip_iteration: int, wait_limit_ns: int = 0) -> None:
    _lib.moe_debug_set_fault(int(skip_iteration), int(wait_limit_ns))


def moe_plan_max_rows(shp: MoeShape) -> int:
    return _lib.moe_plan_max_rows(ctypes.byref(shp))


def moe_plan_export(shp, workspace, stream=None) -> dict:
    import numpy as np
    E, R = shp.E, shp.T * shp.topk
    counts = np.zeros(E, np.int32)
    offs = np.zeros(E + 1, np.int32)
    poffs = np.zeros(E + 1, np.int32)
    row_of = np.zeros(max(R, 1), np.int32)
    src_of = np.zeros(max(moe_plan_max_rows(shp), 1), np.int32)
    P = ctypes.c_int32(0)
    _check("moe_plan_export", _lib.moe_plan_export(
        ctypes.byref(shp), _ptr(workspace), counts.ctypes.data, offs.ctypes.data,
        poffs.ctypes.data, row_of.ctypes.data, src_of.ctypes.data, ctypes.addressof(P),
        _stream(stream)))
    return dict(counts=counts, offs=offs, poffs=poffs, row_of=row_of[:R].reshape(shp.T, shp.topk),
                src_of=src_of[:P.value].copy(), P=P.value)


_timing_keep = None


def moe_set_timing_events(events) -> None:
    """events: five torch.cuda.Event (already recorded once, so they exist)
    or None to stop recording."""
    global _timing_keep
    if events is None:
        _timing_keep = None
        _lib.moe_set_timing_events(None, 0)
        return
    arr = (_vp * len(events))(*[e.cuda_event for e in events])
    _timing_keep = (arr, events)
    _lib.moe_set_timing_events(arr, len(events))


def moe_debug_requant(a, codes, sbytes, stream=None):
    rows, cols = a.shape
    _check("moe_debug_requant", _lib.moe_debug_requant(_ptr(a), rows, cols, _ptr(codes),
                                                       _ptr(sbytes), _stream(stream)))


def moe_gemm_b_bytes(G: int, N: int, K: int):
    sf = _sz(0)
    n = _lib.moe_gemm_b_bytes(G, N, K, ctypes.byref(sf))
    return n, sf.value


def moe_gemm_transform_b(G, N, K, b, b_sf, b_t, b_sf_t, stream=None):
    _check("moe_gemm_transform_b", _lib.moe_gemm_transform_b(
        G, N, K, _ptr(b), _ptr(b_sf), _ptr(b_t), _ptr(b_sf_t), _stream(stream)))


def moe_gemm_workspace_bytes(G: int, M_max: int, N: int, K: int) -> int:
    return _lib.moe_gemm_workspace_bytes(G, M_max, N, K)


def moe_gemm_fp8_fp4(M, N, K, a, a_sf, b_t, b_sf_t, d, workspace, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check("moe_gemm_fp8_fp4", _lib.moe_gemm_fp8_fp4(
        M, N, K, _ptr(a), _ptr(a_sf), _ptr(b_t), _ptr(b_sf_t), _ptr(d), _ptr(workspace),
        ws_bytes, _stream(stream)))


def moe_gemm_fp8_fp4_masked(G, M_max, N, K, a, a_sf, masked_m, b_t, b_sf_t, d, workspace,
                            ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check("moe_gemm_fp8_fp4_masked", _lib.moe_gemm_fp8_fp4_masked(
        G, M_max, N, K, _ptr(a), _ptr(a_sf), _ptr(masked_m), _ptr(b_t), _ptr(b_sf_t), _ptr(d),
        _ptr(workspace), ws_bytes, _stream(stream)))


# ------------------------------------------------------- torch conveniences
def transform_weights(shp, w1, w1_sf, w2, w2_sf, stream=None):
    """Allocate the transformed weight buffers (torch, on w1's device) and
    run moe_transform_weights.  Returns (w1_t, w1_sf_t, w2_t, w2_sf_t)."""
    import torch
    dev = w1.device
    n1, s1 = moe_transformed_bytes(shp, 1)
    n2, s2 = moe_transformed_bytes(shp, 2)
    outs = [torch.empty(n, dtype=torch.uint8, device=dev) for n in (n1, s1, n2, s2)]
    moe_transform_weights(shp, w1, w1_sf, w2, w2_sf, *outs, stream=stream)
    return tuple(outs)


def alloc_workspace(shp, device, host_variant=False):
    """host_variant: False (moe_plan / moe_forward), True (moe_forward_host) or
    "pipelined" (moe_forward_host_pipelined)."""
    import torch
    if host_variant == "pipelined":
        n = moe_workspace_bytes_host_pipelined(shp)
    elif host_variant:
        n = moe_workspace_bytes_host(shp)
    else:
        n = moe_workspace_bytes(shp)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def gemm_transform_b(G, N, K, b, b_sf, stream=None):
    """Allocate the transformed B buffers (torch, on b's device) and run
    moe_gemm_transform_b.  Returns (b_t, b_sf_t)."""
    import torch
    n, sfn = moe_gemm_b_bytes(G, N, K)
    outs = [torch.empty(max(v, 256), dtype=torch.uint8, device=b.device) for v in (n, sfn)]
    moe_gemm_transform_b(G, N, K, b, b_sf, *outs, stream=stream)
    return tuple(outs)


def alloc_gemm_workspace(G, M_max, N, K, device):
    import torch
    n = moe_gemm_workspace_bytes(G, M_max, N, K)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


# ------------------------------------------------------------ FP4 indexer
def moe_mqa_logits_workspace_bytes(S: int, Hh: int, D: int, N: int) -> int:
    return _lib.moe_mqa_logits_workspace_bytes(S, Hh, D, N)


def moe_fp8_fp4_mqa_logits(q, q_sf, kv, kv_sf, weights, ks, ke, logits, workspace, clean=True,
                           ws_bytes=None, stream=None):
    """logits [S, N] (fp32, device) of FP8 queries q [S, Hh, D] against FP4
    keys kv [N, D/2]; see include/moe.h for the layouts."""
    S, Hh, D = q.shape
    N = kv.shape[0]
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check("moe_fp8_fp4_mqa_logits", _lib.moe_fp8_fp4_mqa_logits(
        S, Hh, D, N, _ptr(q), _ptr(q_sf), _ptr(kv), _ptr(kv_sf), _ptr(weights), _ptr(ks),
        _ptr(ke), 1 if clean else 0, _ptr(logits), _ptr(workspace), ws_bytes, _stream(stream)))


def alloc_mqa_workspace(S, Hh, D, N, device):
    import torch
    n = moe_mqa_logits_workspace_bytes(S, Hh, D, N)
    if n == 0:
        raise MoeError("moe_mqa_logits_workspace_bytes", 2)
    return torch.empty(n, dtype=torch.uint8, device=device)
