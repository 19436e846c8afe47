"""Helpers shared by the GPU tests: move synthetic inputs to the device, run
the library through its C ABI, compare with the oracle."""
from __future__ import annotations

import numpy as np

TOL_NORM = 5e-3      # normwise relative error bound on y
TOL_ELEM = 2e-2      # per element: |dy| <= TOL_ELEM * (|y_ref| + rms(y_ref))


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def parity(y_gpu_bits: np.ndarray, y_ref_bits: np.ndarray) -> dict:
    yg = bf16_bits_to_f32(y_gpu_bits).astype(np.float64)
    yr = bf16_bits_to_f32(y_ref_bits).astype(np.float64)
    d = yg - yr
    rms = float(np.sqrt((yr ** 2).mean())) if yr.size else 0.0
    norm = float(np.linalg.norm(d) / max(np.linalg.norm(yr), 1e-300)) if yr.size else 0.0
    elem = float((np.abs(d) / (np.abs(yr) + rms + 1e-300)).max()) if yr.size else 0.0
    return dict(norm=norm, elem=elem, nonfinite=int((~np.isfinite(yg)).sum()),
                exact_frac=float((y_gpu_bits == y_ref_bits).mean()) if yr.size else 1.0)


def assert_parity(y_gpu_bits, y_ref_bits, label=""):
    p = parity(y_gpu_bits, y_ref_bits)
    assert p["nonfinite"] == 0, (label, p)
    assert p["norm"] <= TOL_NORM, (label, p)
    assert p["elem"] <= TOL_ELEM, (label, p)
    return p


class Layer:
    """Inputs of one workload on the device plus its transformed weights."""

    def __init__(self, inputs: dict, device="cuda"):
        import torch

        import block_scaled_fp8_permute_b200 as moe
        self.moe = moe
        self.np = inputs
        T, H = inputs["x"].shape
        E, twoI, _ = inputs["w1"].shape
        k = inputs["topk_idx"].shape[1]
        self.shape = moe.shape(T, H, twoI // 2, E, k)
        self.dev = {key: torch.from_numpy(np.ascontiguousarray(v)).to(device)
                    for key, v in inputs.items()}
        d = self.dev
        self.wt = moe.transform_weights(self.shape, d["w1"], d["w1_sf"], d["w2"], d["w2_sf"])
        self.ws = moe.alloc_workspace(self.shape, device)
        self.y = torch.empty((max(T, 1), H), dtype=torch.bfloat16, device=device)

    def run(self, topk_idx=None, topk_w=None, x=None, x_sf=None):
        d = self.dev
        idx = d["topk_idx"] if topk_idx is None else topk_idx
        self.moe.moe_plan(self.shape, idx, self.ws)
        self.moe.moe_forward(self.shape, d["x"] if x is None else x,
                             d["x_sf"] if x_sf is None else x_sf, idx,
                             d["topk_w"] if topk_w is None else topk_w, *self.wt, self.y,
                             self.ws)
        return self

    def y_bits(self) -> np.ndarray:
        import torch
        torch.cuda.synchronize()
        T = self.shape.T
        return self.y[:T].view(torch.int16).cpu().numpy().view(np.uint16)

    def status(self) -> int:
        return self.moe.moe_get_device_status(self.ws)
