"""Pins for the float64 oracle: each check ties it to something other than itself.

Sources of truth used here: the printed E2M1 value list (golden file), the
bit-field definition of FP4 E2M1 and E8M0, the ml_dtypes / torch decoders
(library routines), numpy / scipy routines, closed forms of special cases, and
the independent NumPy dense brute force (all experts, then masked).
"""

import math
import os

import ml_dtypes
import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import dense_ref
from gen.synth import CONFIGS, Config, f32_to_bf16_bits, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_e2m1():
    vals = {}
    with open(os.path.join(GOLDEN, "e2m1_values.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            c, v = line.split()
            vals[int(c)] = float(v)
    return [vals[c] for c in range(16)]


def _e2m1_from_bits(code):
    """FP4 E2M1 from its bit fields: sign, 2-bit exponent with bias 1, 1-bit mantissa."""
    s = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1.0 + 0.5 * m)
    return math.copysign(mag, s)


# ---------------------------------------------------------------- dequantisation


def test_e2m1_table_matches_printed_list_bits_and_ml_dtypes():
    golden = _golden_e2m1()
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for c in range(16):
        v = oracle.e2m1_value(c)
        assert v == golden[c] == _e2m1_from_bits(c) == lib[c]
        assert math.copysign(1.0, v) == math.copysign(1.0, golden[c])  # -0 for code 8
    assert sorted({abs(v) for v in golden}) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e8m0_scale_is_power_of_two():
    s = np.arange(0, 255, dtype=np.uint8)
    lib = s.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    tch = torch.from_numpy(s.copy()).view(torch.float8_e8m0fnu).double().numpy()
    for i in range(255):
        assert oracle.e8m0_value(i) == 2.0 ** (i - 127) == lib[i] == tch[i]


def test_dequant_exhaustive_bytes_and_scales_bf16_exact():
    """Every byte 0..255 under every scale 2..252, as bf16 bits, against ml_dtypes."""
    scales_range = np.arange(2, 253, dtype=np.uint8)
    nb = 16  # 16 blocks x 16 bytes = 256 bytes per row: one row holds every byte value
    blocks = np.broadcast_to(np.arange(256, dtype=np.uint8).reshape(1, nb, 16), (scales_range.size, nb, 16))
    scales = np.broadcast_to(scales_range[:, None], (scales_range.size, nb))
    bits, inexact = oracle.dequant_bf16(blocks, scales)
    assert inexact == 0
    # library reference: decode codes and scale, multiply in float64, cast to bfloat16
    lo = blocks & 15
    hi = blocks >> 4
    codes = np.stack([lo, hi], -1).reshape(scales_range.size, nb * 32)
    v = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    sc = np.repeat(scales.view(ml_dtypes.float8_e8m0fnu).astype(np.float64), 32, axis=1)
    ref = (v * sc).astype(ml_dtypes.bfloat16)
    assert np.array_equal(bits, ref.view(np.uint16))
    # the product is exact: widening the bf16 back recovers the float64 value
    assert np.array_equal(ref.astype(np.float64), v * sc)
    # -0 survives as 0x8000 for code 8 (byte 0x08 low nibble, 0x80 high nibble)
    assert bits[0, 2 * 0x08] == 0x8000 and bits[0, 2 * 0x80 + 1] == 0x8000


def test_dequant_out_of_contract_scales_are_flagged():
    blocks = np.full((1, 1, 16), 0x11, np.uint8)  # 0.5 everywhere
    _, bad1 = oracle.dequant_bf16(blocks, np.array([[1]], np.uint8))  # 0.5 * 2^-126 is subnormal
    _, bad2 = oracle.dequant_bf16(np.full((1, 1, 16), 0x77, np.uint8), np.array([[254]], np.uint8))  # 6*2^127 = inf
    assert bad1 == 32 and bad2 == 32


@pytest.mark.parametrize("R,C", [(3, 64), (2, 96)])
def test_dequant_placement_low_nibble_first(R, C):
    """A single nonzero nibble at (r, c) must land at exactly (r, c)."""
    nb = C // 32
    scales = np.full((R, nb), 127, np.uint8)
    for r in range(R):
        for c in range(C):
            blocks = np.zeros((R, nb, 16), np.uint8)
            code = 2  # 1.0
            byte = code if c % 2 == 0 else code << 4
            blocks[r, c // 32, (c % 32) // 2] = byte
            d = oracle.dequant(blocks, scales)
            nz = np.argwhere(d != 0)
            assert nz.tolist() == [[r, c]] and d[r, c] == 1.0


def test_dequant_matches_dense_decoder_random():
    rng = np.random.default_rng(5)
    blocks = rng.integers(0, 256, (7, 4, 16), dtype=np.uint8)
    scales = rng.integers(100, 140, (7, 4), dtype=np.uint8)
    assert np.array_equal(oracle.dequant(blocks, scales), dense_ref.dequant_bank(blocks, scales))


# ---------------------------------------------------------------- router


def test_bf16_input_widening_matches_library():
    rng = np.random.default_rng(1)
    f = rng.standard_normal(1000).astype(np.float32) * 10
    bits = f32_to_bf16_bits(f)
    assert np.array_equal(bits, f.astype(ml_dtypes.bfloat16).view(np.uint16))  # RNE, like ml_dtypes
    rw = np.eye(1000, dtype=np.float32)[:3]
    lg = oracle.router_logits(bits[None, :], rw, np.zeros(3, np.float32))
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()[:3]
    assert np.array_equal(lg[0], ref)


def test_router_logits_match_numpy_matmul():
    rng = np.random.default_rng(2)
    T, H, E = 9, 200, 13
    x = f32_to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    rw = rng.standard_normal((E, H), dtype=np.float32)
    rb = rng.standard_normal(E, dtype=np.float32)
    ref = x.view(ml_dtypes.bfloat16).astype(np.float64) @ rw.astype(np.float64).T + rb.astype(np.float64)
    np.testing.assert_allclose(oracle.router_logits(x, rw, rb), ref, rtol=1e-12, atol=1e-12)


def test_topk_matches_stable_argsort_and_softmax():
    rng = np.random.default_rng(3)
    lg = rng.standard_normal((50, 17))
    for k in (1, 2, 4, 17):
        idx, w = oracle.topk_softmax(lg, k)
        ref_idx = np.argsort(-lg, axis=1, kind="stable")[:, :k]
        assert np.array_equal(idx, ref_idx)
        sel = np.take_along_axis(lg, ref_idx, 1)
        np.testing.assert_allclose(w, scipy.special.softmax(sel, axis=1), rtol=1e-13)
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-14)
        if k == 1:
            assert np.all(w == 1.0)
        if k == 17:  # k == E: the full softmax over all experts, in descending order
            np.testing.assert_allclose(np.sort(w, 1)[:, ::-1], np.sort(scipy.special.softmax(lg, 1), 1)[:, ::-1],
                                       rtol=1e-13)


def test_topk_exact_tie_goes_to_lower_index():
    lg = np.array([[0.5, 2.0, 1.0, 2.0, 1.0]])
    idx, w = oracle.topk_softmax(lg, 3)
    assert idx.tolist() == [[1, 3, 2]]
    assert w[0, 0] == w[0, 1]


def test_router_margin_definition():
    # logits = bias only (x is zero): sorted 3.0, 2.5, 2.499, 1.0 -> k=2 looks at the top 3
    rb = np.array([1.0, 2.5, 3.0, 2.499], np.float32)
    x = np.zeros((1, 32), np.uint16)
    m = oracle.router_margins(x, np.zeros((4, 32), np.float32), rb, 2, threads=1)
    assert abs(m[0] - (np.float64(np.float32(2.5)) - np.float64(np.float32(2.499)))) < 1e-12
    m1 = oracle.router_margins(x, np.zeros((4, 32), np.float32), rb, 1, threads=1)
    assert abs(m1[0] - 0.5) < 1e-12


# ---------------------------------------------------------------- activation, interleave


def _mini_inputs(T=2, H=64, I=64, E=3, seed=0):
    cfg = Config("mini", T=T, H=H, I=I, E=E, k=2, scale_lo=120, scale_hi=124, router_bias="normal")
    return cfg, make_inputs(cfg, seed=seed)


def _bf16(v):
    return f32_to_bf16_bits(np.asarray(v, np.float32))


def test_clamp_points_and_one_sided_gate():
    """Zero weight bytes make h equal to the bias exactly; walk gate/up over the clamp points."""
    pts = np.array([-100.0, -7.5, -7.0, 0.0, 6.96875, 7.0, 7.5, 100.0])
    assert np.array_equal(_bf16(pts).view(ml_dtypes.bfloat16).astype(np.float64), pts)  # exactly representable
    n = pts.size
    I = 32 * ((n * n + 31) // 32)
    H = 32
    g, u = np.meshgrid(pts, pts, indexing="ij")
    g, u = g.ravel(), u.ravel()
    bias = np.zeros(2 * I)
    bias[0:2 * g.size:2] = g
    bias[1:2 * g.size:2] = u
    inputs = {
        "gate_up_blocks": np.zeros((1, 2 * I, H // 32, 16), np.uint8),
        "gate_up_scales": np.full((1, 2 * I, H // 32), 127, np.uint8),
        "gate_up_bias": _bf16(bias)[None],
        "down_blocks": np.zeros((1, H, I // 32, 16), np.uint8),
        "down_scales": np.full((1, H, I // 32), 127, np.uint8),
        "down_bias": np.zeros((1, H), np.uint16),
    }
    h, a, y = oracle.expert(np.ones(H), inputs, 0)
    assert np.array_equal(h, bias)
    a = a[: g.size].reshape(n, n)  # [gate point, up point]
    gi = {v: i for i, v in enumerate(pts)}
    # gate is clamped from above at 7: 7, 7.5 and 100 give the same row
    assert np.array_equal(a[gi[7.0]], a[gi[7.5]]) and np.array_equal(a[gi[7.0]], a[gi[100.0]])
    # up is clamped to [-7, 7]: columns at -100/-7.5/-7 agree, and 7/7.5/100 agree
    assert np.array_equal(a[:, gi[-7.0]], a[:, gi[-7.5]]) and np.array_equal(a[:, gi[-7.0]], a[:, gi[-100.0]])
    assert np.array_equal(a[:, gi[7.0]], a[:, gi[7.5]]) and np.array_equal(a[:, gi[7.0]], a[:, gi[100.0]])
    # gate has no lower clamp: -100 differs from -7.5 and -7
    assert not np.allclose(a[gi[-100.0]], a[gi[-7.0]], rtol=0, atol=1e-12)
    # special cases: gate 0 -> 0; up -1 would give 0 (u+1 factor)
    assert np.all(a[gi[0.0]] == 0.0)
    # closed forms with mpmath at 50 digits
    import mpmath
    mpmath.mp.dps = 50

    def ref(gv, uv):
        gv = min(gv, 7.0)
        uv = max(min(uv, 7.0), -7.0)
        return float((mpmath.mpf(uv) + 1) * gv / (1 + mpmath.exp(-mpmath.mpf("1.702") * gv)))

    for i, gv in enumerate(pts):
        for j, uv in enumerate(pts):
            # rel 1e-12: at g = -100 the rounding of 1.702*g (about 1e-14 absolute) moves exp(170.2) by ~1e-14 relative
            assert a[i, j] == pytest.approx(ref(gv, uv), rel=1e-12, abs=1e-300)
    # e.g. g = 100 -> 7 * sigmoid(11.914); u = -100 -> -7 -> factor (-6)
    assert a[gi[100.0], gi[-100.0]] == pytest.approx(-6 * 7 / (1 + math.exp(-11.914)), rel=1e-14)


def test_interleave_gate_rows_even_up_rows_odd():
    """gate = rows 0::2, up = rows 1::2 of the interleaved gate_up; swapping the reading is detectably wrong."""
    I, H = 32, 32
    rng = np.random.default_rng(7)
    gate_b = rng.uniform(-3, 3, I)
    up_b = rng.uniform(-3, 3, I)
    bias = np.empty(2 * I)
    bias[0::2], bias[1::2] = gate_b, up_b
    bias = _bf16(bias).view(ml_dtypes.bfloat16).astype(np.float64)
    gate_b, up_b = bias[0::2], bias[1::2]
    inputs = {
        "gate_up_blocks": np.zeros((1, 2 * I, 1, 16), np.uint8),
        "gate_up_scales": np.full((1, 2 * I, 1), 127, np.uint8),
        "gate_up_bias": _bf16(bias)[None],
        "down_blocks": np.zeros((1, H, 1, 16), np.uint8),
        "down_scales": np.full((1, H, 1), 127, np.uint8),
        "down_bias": np.zeros((1, H), np.uint16),
    }
    _, a, _ = oracle.expert(np.zeros(H), inputs, 0)
    sig = scipy.special.expit
    right = (up_b + 1) * gate_b * sig(1.702 * gate_b)
    swapped = (gate_b + 1) * up_b * sig(1.702 * up_b)
    np.testing.assert_allclose(a, right, rtol=1e-13)
    assert np.abs(a - swapped).max() > 0.1


def test_interleave_through_weights_one_hot():
    """Row r of gate_up with a single code at column c: one-hot x selects W[r, c]."""
    I, H = 32, 64
    blocks = np.zeros((1, 2 * I, H // 32, 16), np.uint8)
    c = 37
    for r in range(2 * I):
        code = 1 + (r % 7)  # 0.5 .. 6
        blocks[0, r, c // 32, (c % 32) // 2] = code << (4 * (c % 2))
    inputs = {
        "gate_up_blocks": blocks,
        "gate_up_scales": np.full((1, 2 * I, H // 32), 126, np.uint8),  # x 0.5
        "gate_up_bias": np.zeros((1, 2 * I), np.uint16),
        "down_blocks": np.zeros((1, H, I // 32, 16), np.uint8),
        "down_scales": np.full((1, H, I // 32), 127, np.uint8),
        "down_bias": np.zeros((1, H), np.uint16),
    }
    x = np.zeros(H)
    x[c] = 1.0
    h, a, _ = oracle.expert(x, inputs, 0)
    golden = _golden_e2m1()
    expect_h = np.array([golden[1 + (r % 7)] * 0.5 for r in range(2 * I)])
    assert np.array_equal(h, expect_h)
    g = np.minimum(expect_h[0::2], 7)
    u = np.clip(expect_h[1::2], -7, 7)
    np.testing.assert_allclose(a, (u + 1) * g * scipy.special.expit(1.702 * g), rtol=1e-14)


def test_sigmoid_matches_scipy():
    for v in (-30.0, -1.0, 0.0, 0.3, 11.914):
        assert oracle.sigmoid(v) == pytest.approx(float(scipy.special.expit(v)), rel=1e-15)


# ---------------------------------------------------------------- whole layer


def test_oracle_equals_dense_brute_force_tiny():
    inp = make_inputs("tiny", margin_fn=oracle.router_margins)
    out, idx, w = oracle.moe_forward(inp, 2)
    o2, i2, w2, _ = dense_ref.forward(inp, 2)
    assert np.array_equal(idx, i2)
    np.testing.assert_allclose(w, w2, rtol=1e-14)
    np.testing.assert_allclose(out, o2, rtol=1e-12, atol=1e-12 * np.abs(o2).max())


def test_oracle_equals_dense_brute_force_T4_E4():
    cfg = Config("t4e4", T=4, H=64, I=96, E=4, k=2, scale_lo=118, scale_hi=126, router_bias="normal")
    inp = make_inputs(cfg, seed=11, margin_fn=oracle.router_margins)
    out, idx, w = oracle.moe_forward(inp, 2)
    o2, i2, w2, _ = dense_ref.forward(inp, 2)
    assert np.array_equal(idx, i2)
    np.testing.assert_allclose(out, o2, rtol=1e-12, atol=1e-12 * np.abs(o2).max())
    # k = E: every expert, weights = full softmax
    out4, idx4, w4 = oracle.moe_forward(inp, 4)
    o24, _, _, _ = dense_ref.forward(inp, 4)
    np.testing.assert_allclose(out4, o24, rtol=1e-12, atol=1e-12 * np.abs(o24).max())


def test_zero_weights_closed_form():
    """All weight bytes zero: y = down_bias, so out = sum_s w_s * down_bias[e_s]."""
    cfg, inp = _mini_inputs(T=5, E=4)
    inp["gate_up_blocks"][:] = 0
    inp["down_blocks"][:] = 0
    out, idx, w = oracle.moe_forward(inp, 2)
    bd = inp["down_bias"].view(ml_dtypes.bfloat16).astype(np.float64)
    ref = np.einsum("ts,tsh->th", w, bd[idx])
    np.testing.assert_allclose(out, ref, rtol=1e-15)


def test_single_expert_layer_is_that_expert():
    """k = 1 gives weight 1 and out = y of the argmax expert."""
    cfg, inp = _mini_inputs(T=3, E=3, seed=4)
    out, idx, w = oracle.moe_forward(inp, 1)
    assert np.all(w == 1.0)
    x64 = inp["x"].view(ml_dtypes.bfloat16).astype(np.float64)
    for t in range(3):
        _, _, y = oracle.expert(x64[t], inp, int(idx[t, 0]))
        assert np.array_equal(out[t], y)


def test_token_subset_and_threads_bit_identical():
    inp = make_inputs("tiny", margin_fn=oracle.router_margins)
    out1, idx1, w1 = oracle.moe_forward(inp, 2, threads=1)
    out4, idx4, w4 = oracle.moe_forward(inp, 2, threads=4)
    assert np.array_equal(out1, out4) and np.array_equal(idx1, idx4)
    sub = [3, 0, 15]
    outs, idxs, _ = oracle.moe_forward(inp, 2, tokens=sub, threads=2)
    assert np.array_equal(outs, out1[sub]) and np.array_equal(idxs, idx1[sub])


def test_linearity_in_down_bias():
    """out is affine in the down bias: adding delta to every expert's bias adds delta * sum_s w_s = delta."""
    cfg, inp = _mini_inputs(T=4, E=3, seed=9)
    out0, idx, w = oracle.moe_forward(inp, 2)
    inp2 = dict(inp)
    bd = inp["down_bias"].view(ml_dtypes.bfloat16).astype(np.float64) + 0.25
    inp2["down_bias"] = f32_to_bf16_bits(bd.astype(np.float32))
    out1, idx1, _ = oracle.moe_forward(inp2, 2)
    bd2 = inp2["down_bias"].view(ml_dtypes.bfloat16).astype(np.float64)
    delta = np.einsum("ts,tsh->th", w, bd2[idx] - inp["down_bias"].view(ml_dtypes.bfloat16).astype(np.float64)[idx])
    np.testing.assert_allclose(out1 - out0, delta, rtol=1e-9, atol=1e-12)
