"""Float64 CPU oracle for the GPT-OSS MXFP4 MoE feed-forward layer.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers. The product library never imports this
package, and this package imports nothing from the product.

Two independent restatements of the same definition live here:

* ``moe_oracle.c`` (loaded through ctypes): the plain per-token loops in
  float64, one term at a time, with an optional OpenMP split over tokens.
* ``dense_ref.py``: a NumPy float64 brute force that evaluates every expert
  on every token and masks to the top-k, decoding FP4/E8M0 through ml_dtypes.

Parity pins: every function here is pinned by a ``-m "not gpu"`` test against
library decoders, closed forms, or the other restatement; none is "parity
unpinned".
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (IEEE double, no contraction, OpenMP over tokens)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_e2m1_value.restype = ctypes.c_double
        lib.oracle_e2m1_value.argtypes = [ctypes.c_int]
        lib.oracle_e8m0_value.restype = ctypes.c_double
        lib.oracle_e8m0_value.argtypes = [ctypes.c_int]
        lib.oracle_sigmoid.restype = ctypes.c_double
        lib.oracle_sigmoid.argtypes = [ctypes.c_double]
        lib.oracle_dequant.restype = None
        lib.oracle_dequant.argtypes = [P, P, I64, I64, P]
        lib.oracle_dequant_bf16.restype = I64
        lib.oracle_dequant_bf16.argtypes = [P, P, I64, I64, P]
        lib.oracle_router_logits.restype = None
        lib.oracle_router_logits.argtypes = [P, P, P, I64, I64, I64, P]
        lib.oracle_topk_softmax.restype = None
        lib.oracle_topk_softmax.argtypes = [P, I64, I64, ctypes.c_int, P, P]
        lib.oracle_router_margins.restype = None
        lib.oracle_router_margins.argtypes = [P, P, P, I64, I64, I64, ctypes.c_int, ctypes.c_int, P]
        lib.oracle_swiglu.restype = None
        lib.oracle_swiglu.argtypes = [P, I64, P]
        lib.oracle_expert.restype = None
        lib.oracle_expert.argtypes = [P, P, P, P, P, P, P, I64, I64, P, P, P]
        lib.oracle_moe_forward.restype = ctypes.c_int
        lib.oracle_moe_forward.argtypes = [P] * 9 + [I64, I64, I64, I64, ctypes.c_int, P, I64, ctypes.c_int, P, P,
                                                     P]
        lib.oracle_has_openmp.restype = ctypes.c_int
        _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def e2m1_value(code: int) -> float:
    return _load().oracle_e2m1_value(int(code))


def e8m0_value(s: int) -> float:
    return _load().oracle_e8m0_value(int(s))


def sigmoid(v: float) -> float:
    return _load().oracle_sigmoid(float(v))


def dequant(blocks: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """MXFP4 [R, C/32, 16] + [R, C/32] -> float64 [R, C]."""
    b = _c(blocks, np.uint8)
    s = _c(scales, np.uint8)
    R, nb = s.shape[-2], s.shape[-1]
    b = b.reshape(-1, nb, 16)
    s = s.reshape(-1, nb)
    R = s.shape[0]
    out = np.empty((R, nb * 32), np.float64)
    _load().oracle_dequant(_p(b), _p(s), R, nb * 32, _p(out))
    return out


def dequant_bf16(blocks: np.ndarray, scales: np.ndarray):
    """MXFP4 -> bf16 bit patterns uint16 [R, C]; also returns the count of inexact elements."""
    b = _c(blocks, np.uint8)
    s = _c(scales, np.uint8)
    nb = s.shape[-1]
    b = b.reshape(-1, nb, 16)
    s = s.reshape(-1, nb)
    R = s.shape[0]
    out = np.empty((R, nb * 32), np.uint16)
    bad = _load().oracle_dequant_bf16(_p(b), _p(s), R, nb * 32, _p(out))
    return out, int(bad)


def router_logits(x: np.ndarray, router_w: np.ndarray, router_b: np.ndarray) -> np.ndarray:
    x = _c(x, np.uint16)
    rw = _c(router_w, np.float32)
    rb = _c(router_b, np.float32)
    T, H = x.shape
    E = rw.shape[0]
    out = np.empty((T, E), np.float64)
    _load().oracle_router_logits(_p(x), _p(rw), _p(rb), T, H, E, _p(out))
    return out


def topk_softmax(logits: np.ndarray, k: int):
    lg = _c(logits, np.float64)
    T, E = lg.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    _load().oracle_topk_softmax(_p(lg), T, E, int(k), _p(idx), _p(w))
    return idx, w


def router_margins(x: np.ndarray, router_w: np.ndarray, router_b: np.ndarray, k: int,
                   threads: int = 0) -> np.ndarray:
    """Per token, the smallest adjacent gap among the k+1 largest logits (float64)."""
    x = _c(x, np.uint16)
    rw = _c(router_w, np.float32)
    rb = _c(router_b, np.float32)
    T, H = x.shape
    E = rw.shape[0]
    out = np.empty(T, np.float64)
    _load().oracle_router_margins(_p(x), _p(rw), _p(rb), T, H, E, int(k), int(threads or os.cpu_count() or 1),
                                  _p(out))
    return out


def swiglu(h: np.ndarray) -> np.ndarray:
    h = _c(h, np.float64).reshape(-1)
    I = h.shape[0] // 2
    out = np.empty(I, np.float64)
    _load().oracle_swiglu(_p(h), I, _p(out))
    return out


def expert(xrow: np.ndarray, inputs: Dict[str, np.ndarray], e: int):
    """One expert on one float64 token row: returns (h [2I], act [I], y [H])."""
    gb = _c(inputs["gate_up_blocks"][e], np.uint8)
    gs = _c(inputs["gate_up_scales"][e], np.uint8)
    gbias = _c(inputs["gate_up_bias"][e], np.uint16)
    db = _c(inputs["down_blocks"][e], np.uint8)
    ds = _c(inputs["down_scales"][e], np.uint8)
    dbias = _c(inputs["down_bias"][e], np.uint16)
    H = db.shape[0]
    I = db.shape[1] * 32
    x = _c(xrow, np.float64)
    h = np.empty(2 * I, np.float64)
    a = np.empty(I, np.float64)
    y = np.empty(H, np.float64)
    _load().oracle_expert(_p(x), _p(gb), _p(gs), _p(gbias), _p(db), _p(ds), _p(dbias), H, I, _p(h), _p(a), _p(y))
    return h, a, y


def moe_forward(inputs: Dict[str, np.ndarray], k: int, tokens: Optional[Sequence[int]] = None,
                threads: int = 1):
    """The layer on all tokens (or a list of token indices).

    Returns (out float64 [n, H], idx int32 [n, k], w float64 [n, k]).
    """
    x = _c(inputs["x"], np.uint16)
    rw = _c(inputs["router_w"], np.float32)
    rb = _c(inputs["router_b"], np.float32)
    gb = _c(inputs["gate_up_blocks"], np.uint8)
    gs = _c(inputs["gate_up_scales"], np.uint8)
    gbias = _c(inputs["gate_up_bias"], np.uint16)
    db = _c(inputs["down_blocks"], np.uint8)
    ds = _c(inputs["down_scales"], np.uint8)
    dbias = _c(inputs["down_bias"], np.uint16)
    T, H = x.shape
    E = rw.shape[0]
    I = db.shape[2] * 32
    tl = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    n = T if tl is None else tl.shape[0]
    out = np.empty((n, H), np.float64)
    idx = np.empty((n, k), np.int32)
    w = np.empty((n, k), np.float64)
    rc = _load().oracle_moe_forward(_p(x), _p(rw), _p(rb), _p(gb), _p(gs), _p(gbias), _p(db), _p(ds), _p(dbias), T,
                                    H, I, E, int(k), _p(tl), n, int(threads), _p(out), _p(idx), _p(w))
    if rc:
        raise ValueError("oracle_moe_forward rejected its arguments")
    return out, idx, w


def has_openmp() -> bool:
    return bool(_load().oracle_has_openmp())
