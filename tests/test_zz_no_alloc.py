"""The allocation-free entry point (moe_forward_noalloc) against the handle-based moe_forward.

moe_forward_noalloc serves callers that cannot allocate device memory where
they run the layer; it keeps its intermediates in a fixed scratch array inside
the library. This file is collected last so that a run stopping at its first
failure has already run every other test; it also passes on its own in a fresh
process (the scratch array's device address is looked up on the first call).
"""

import numpy as np
import pytest
import torch

import oracle
from gen.synth import CONFIGS, Config, make_inputs
from tests.gpu_util import MAX_ABS, MAX_REL_TO_PEAK, MEAN_REL, bf16_dev_to_f64, run_forward, score, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from mxfp4_expert_ffn_bias_b200 import build
    build.build()
    from mxfp4_expert_ffn_bias_b200 import moe as m
    torch.cuda.set_device(0)
    return m


def _noalloc(moe, dev, cfg, T):
    out = torch.empty((T, cfg.H), dtype=torch.bfloat16, device="cuda")
    moe.moe_forward_noalloc(dev["x"], dev["router_w"], dev["router_b"], dev["gate_up_blocks"], dev["gate_up_scales"],
                            dev["gate_up_bias"], dev["down_blocks"], dev["down_scales"], dev["down_bias"], cfg.H,
                            cfg.I, cfg.E, cfg.k, T, out)
    return out


@pytest.mark.parametrize("cfg", [CONFIGS["gpt-oss-20b-decode"], CONFIGS["tiny"],
                                 Config("no-alloc-16x4", T=16, H=2880, I=2880, E=128, k=4, scale_lo=118,
                                        scale_hi=122, router_bias="normal")], ids=lambda c: c.name)
def test_noalloc_matches_moe_forward_twice(moe, cfg):
    inp = make_inputs(cfg, seed=3, margin_fn=oracle.router_margins)
    dev = to_device(inp)
    T = inp["x"].shape[0]
    h = moe.moe_create(cfg.H, cfg.I, cfg.E, cfg.k, T)
    try:
        ref = bf16_dev_to_f64(run_forward(moe, h, dev, T, cfg.H))
    finally:
        moe.moe_destroy(h)
    for _ in range(2):  # two calls in a row share (and reuse) the scratch array
        got = bf16_dev_to_f64(_noalloc(moe, dev, cfg, T))
        torch.cuda.synchronize()
        s = score(got, ref)
        assert s["max_err"] <= MAX_REL_TO_PEAK * s["max_ref"] + MAX_ABS, s
        assert s["mean_rel"] <= MEAN_REL, s


def test_noalloc_rejects_shapes_beyond_its_scratch(moe):
    cfg = CONFIGS["gpt-oss-20b-decode"]
    dev = to_device(make_inputs(cfg, seed=0))
    out = torch.empty((32, cfg.H), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as ei:  # 32 tokens x top-4 = 128 routed rows > 64
        moe.moe_forward_noalloc(dev["x"], dev["router_w"], dev["router_b"], dev["gate_up_blocks"],
                                dev["gate_up_scales"], dev["gate_up_bias"], dev["down_blocks"], dev["down_scales"],
                                dev["down_bias"], cfg.H, cfg.I, cfg.E, cfg.k, 32, out)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
