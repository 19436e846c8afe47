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


def Layer(inputs: dict, device="cuda"):
    """The package's device-resident layer (imported here, not at module load, so
    that collecting the GPU tests on a machine without the built library works)."""
    from block_scaled_fp8_permute_b200.layer import MoELayer
    return MoELayer(inputs, device=device)
