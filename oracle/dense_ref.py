"""NumPy float64 brute force of the GPT-OSS MXFP4 MoE layer (test infrastructure only).

A second, independent restatement of the layer used to cross-check the C
oracle: it decodes FP4 E2M1 codes and E8M0 scales with ml_dtypes (not with the
oracle's value table), dequantises the whole expert bank, evaluates EVERY
expert on EVERY token with dense einsums, and only then masks the result to
each token's top-k experts. This is the "full bank" evaluation that the
ZeroModels GPT-OSS docs ("MXFP4 experts" bullet) say gives the same result as
evaluating only the routed experts.

Memory grows as T * E * max(2I, H); it is meant for tiny layers.
"""

from __future__ import annotations

from typing import Dict, Tuple

import ml_dtypes
import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(bits, dtype=np.uint16).view(ml_dtypes.bfloat16).astype(np.float64)


def dequant_bank(blocks: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """[..., R, C/32, 16] uint8 + [..., R, C/32] uint8 -> float64 [..., R, C]."""
    lo = blocks & np.uint8(0x0F)
    hi = blocks >> np.uint8(4)
    codes = np.stack([lo, hi], axis=-1).reshape(blocks.shape[:-1] + (32,))  # low nibble = even column
    vals = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    sc = np.ascontiguousarray(scales).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    full = vals * sc[..., None]
    return full.reshape(full.shape[:-2] + (full.shape[-2] * 32,))


def route(x64: np.ndarray, rw: np.ndarray, rb: np.ndarray, k: int) -> Tuple[np.ndarray, np.ndarray]:
    logits = x64 @ rw.astype(np.float64).T + rb.astype(np.float64)
    E = logits.shape[1]
    # sort by (-logit, index): lexsort keys are applied last-first
    order = np.lexsort((np.broadcast_to(np.arange(E), logits.shape), -logits), axis=1)
    idx = order[:, :k]
    sel = np.take_along_axis(logits, idx, axis=1)
    ex = np.exp(sel - sel[:, :1])
    return idx.astype(np.int32), ex / ex.sum(axis=1, keepdims=True)


def forward(inputs: Dict[str, np.ndarray], k: int):
    """Returns (out [T, H], idx [T, k], w [T, k], act_all [T, E, I])."""
    x64 = bf16_bits_to_f64(inputs["x"])
    idx, w = route(x64, inputs["router_w"], inputs["router_b"], k)
    wgu = dequant_bank(inputs["gate_up_blocks"], inputs["gate_up_scales"])  # [E, 2I, H]
    wd = dequant_bank(inputs["down_blocks"], inputs["down_scales"])  # [E, H, I]
    bgu = bf16_bits_to_f64(inputs["gate_up_bias"])  # [E, 2I]
    bd = bf16_bits_to_f64(inputs["down_bias"])  # [E, H]
    h = np.einsum("th,erh->ter", x64, wgu) + bgu[None]  # [T, E, 2I]
    gate = np.minimum(h[..., 0::2], 7.0)
    up = np.clip(h[..., 1::2], -7.0, 7.0)
    act = (up + 1.0) * gate / (1.0 + np.exp(-1.702 * gate))
    y = np.einsum("tei,ehi->teh", act, wd) + bd[None]  # [T, E, H]
    T = x64.shape[0]
    ysel = y[np.arange(T)[:, None], idx]  # [T, k, H]
    out = np.einsum("ts,tsh->th", w, ysel)
    return out, idx, w, act
