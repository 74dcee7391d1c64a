"""GPU parity of ssd_bidir_fwd_dtraw: the step size prepared in the kernel from
the raw projection (dt = clamp(softplus(dt_raw + dt_bias), dt_min, dt_max))
against the fp64 oracle's dt_prep followed by its mixer (tolerances in
paritylib)."""
import math

import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as si
from paritylib import check
from ssd_inputs import to_f64

pytestmark = pytest.mark.gpu

# (batch, L, H, N, G): ragged tails, shared and per-head B/C, 8 to 512 units; the
# 64 x 128 row runs the one-tile kernel that reuses shared C/B tiles
SHAPES = [(2, 384, 4, 128, 4), (3, 200, 6, 64, 2), (40, 256, 4, 128, 4), (64, 128, 8, 128, 2), (1, 1, 2, 64, 1)]
LIMITS = [(0.0, math.inf), (1e-3, 0.1), (0.01, 0.05)]


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_b200 as m
    return m


@pytest.mark.parametrize("limits", LIMITS, ids=["unbounded", "1e-3_0.1", "clamped_0.01_0.05"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b%d_L%d_H%d_N%d_G%d" % s)
def test_dtraw_against_oracle(ssd, shape, limits):
    batch, L, H, N, G = shape
    lo, hi = limits
    inp = si.bidir_inputs(batch, L, H, 64, N, G, "bf16", seed=L + H, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(batch * 7 + L)
    # raw projections around softplus^-1 of the usual step sizes, per-head biases
    dt_raw = (torch.randn(2, batch, L, H, device="cuda", generator=gen) - 4.0).to(torch.bfloat16).contiguous()
    bias = (torch.rand(2, H, device="cuda", generator=gen) * 2 - 1).contiguous()
    y = ssd.ssd_bidir_fwd_dtraw(inp["x"], dt_raw, bias, inp["A"], inp["B"], inp["C"], inp["D"], lo, hi)
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    dt = oracle.dt_prep(to_f64(dt_raw), to_f64(bias), lo, hi)
    o = oracle.bidir(to_f64(inp["x"]), dt, to_f64(inp["A"]), to_f64(inp["B"]), to_f64(inp["C"]), to_f64(inp["D"]))
    check(to_f64(y), o, torch.bfloat16, f"dtraw {shape} {limits}")
