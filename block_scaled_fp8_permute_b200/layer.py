"""A device-resident MoE layer over the C ABI: the canonical inputs moved to
one device, the weights transformed once, a workspace and an output buffer.

Convenience around moe_transform_weights / moe_plan / moe_forward: it
allocates with torch and marshals arguments; every step of the layer runs in
libmoe's kernels.
"""
from __future__ import annotations

import numpy as np


ACTIVATIONS = ("x", "x_sf", "topk_idx", "topk_w")
WEIGHTS = ("w1", "w1_sf", "w2", "w2_sf")


class MoELayer:
    """inputs: dict of canonical host arrays (numpy) x, x_sf, topk_idx,
    topk_w, w1, w1_sf, w2, w2_sf (layouts as in include/moe.h).

    The raw weights are copied to the device, transformed once
    (moe_transform_weights) and dropped.  `weights` may instead pass the four
    transformed device tensors of another layer of the same shape (the raw
    weights in `inputs` are then not needed)."""

    def __init__(self, inputs: dict, device="cuda", weights=None):
        import torch

        from . import alloc_workspace, shape, transform_weights
        self.np = inputs
        T, H = inputs["x"].shape
        k = inputs["topk_idx"].shape[1]
        if weights is None:
            E, two_i, _ = inputs["w1"].shape
        else:
            E, two_i = inputs["E"], 2 * inputs["I"]
        self.shape = shape(T, H, two_i // 2, E, k)
        self.dev = {key: torch.from_numpy(np.ascontiguousarray(inputs[key])).to(device)
                    for key in ACTIVATIONS}
        if weights is None:
            raw = [torch.from_numpy(np.ascontiguousarray(inputs[key])).to(device)
                   for key in WEIGHTS]
            self.wt = transform_weights(self.shape, *raw)
            torch.cuda.synchronize(device)
            del raw
        else:
            self.wt = tuple(weights)
        self.ws = alloc_workspace(self.shape, device)
        self.y = torch.empty((max(T, 1), H), dtype=torch.bfloat16, device=device)

    def run(self, topk_idx=None, topk_w=None, x=None, x_sf=None, stream=None):
        """moe_plan + moe_forward on the stored (or the given) device inputs."""
        from . import moe_forward, moe_plan
        d = self.dev
        idx = d["topk_idx"] if topk_idx is None else topk_idx
        moe_plan(self.shape, idx, self.ws, stream=stream)
        moe_forward(self.shape, d["x"] if x is None else x, d["x_sf"] if x_sf is None else x_sf,
                    idx, d["topk_w"] if topk_w is None else topk_w, *self.wt, self.y, self.ws,
                    stream=stream)
        return self

    def y_bits(self) -> np.ndarray:
        """y of the last run as BF16 bit patterns (host uint16 [T, H]); synchronises."""
        import torch
        torch.cuda.synchronize()
        return self.y[:self.shape.T].view(torch.int16).cpu().numpy().view(np.uint16)

    def status(self) -> int:
        from . import moe_get_device_status
        return moe_get_device_status(self.ws)
