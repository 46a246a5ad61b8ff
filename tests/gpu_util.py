"""Helpers shared by the GPU parity tests: upload inputs, run the layer through the C ABI, score outputs."""

from __future__ import annotations

import numpy as np
import torch

# The parity bar for layer outputs (bf16 out vs float64 oracle).
MAX_REL_TO_PEAK = 2e-2   # max|gpu - ref| <= 2e-2 * max|ref| + 1e-3
MAX_ABS = 1e-3
MEAN_REL = 5e-3          # sum|gpu - ref| / sum|ref| (L1-relative)


def to_device(inputs: dict, device="cuda") -> dict:
    d = {}
    for k, v in inputs.items():
        if v.dtype == np.uint16:
            d[k] = torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).to(device)
        else:
            d[k] = torch.from_numpy(np.ascontiguousarray(v)).to(device)
    return d


def bf16_dev_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.bfloat16).float().cpu().numpy().astype(np.float64)


def run_forward(moe, h, dev: dict, T: int, H: int, stream=None) -> torch.Tensor:
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(h, dev["x"], dev["router_w"], dev["router_b"], dev["gate_up_blocks"], dev["gate_up_scales"],
                    dev["gate_up_bias"], dev["down_blocks"], dev["down_scales"], dev["down_bias"], T, out, stream)
    return out


def score(gpu: np.ndarray, ref: np.ndarray) -> dict:
    err = np.abs(gpu - ref)
    return {
        "max_err": float(err.max()),
        "max_ref": float(np.abs(ref).max()),
        "mean_rel": float(err.sum() / max(np.abs(ref).sum(), 1e-300)),
    }


def assert_parity(gpu: np.ndarray, ref: np.ndarray, what: str = "") -> dict:
    s = score(gpu, ref)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite output"
    assert s["max_err"] <= MAX_REL_TO_PEAK * s["max_ref"] + MAX_ABS, f"{what}: {s}"
    assert s["mean_rel"] <= MEAN_REL, f"{what}: {s}"
    return s
