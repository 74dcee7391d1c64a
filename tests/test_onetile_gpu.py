"""GPU parity of the one-tile kernel (ssd_bidir_fwd with SSD_PATH_ONETILE:
sequences of at most 128 tokens, C B^T of each direction computed once per
B/C group and reused for the group's heads) against the fp64 oracle's
bidirectional mixer (oracle.bidir), element by element.

Shapes cover full and ragged tiles (128, 100, 77 and 1 tokens), d_state 64
and 128, B/C shared by all heads, by groups of heads and per head, more
(batch, head) units than SMs (each CTA's run of heads then crosses batch and
group boundaries), decays from mild to extreme, and the packed 128-token
workload at full size on sampled units. Tolerance: paritylib's bf16 bar.
"""
import pytest
import torch

import oracle
import ssd_inputs as si
from paritylib import check, oracle_units, sample_units
from ssd_inputs import to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_b200 as m
    return m


def run(ssd, inp):
    out = ssd.ssd_bidir_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                            path=ssd.SSD_PATH_ONETILE)
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    return out


def full_oracle(inp):
    return oracle.bidir(*(to_f64(inp[k]) for k in ("x", "dt", "A", "B", "C", "D")))


# (batch, L, H, N, G)
SHAPES = [(3, 128, 4, 128, 1), (2, 100, 6, 64, 2), (5, 1, 2, 128, 1), (4, 77, 8, 128, 8),
          (40, 128, 24, 128, 1), (64, 128, 8, 128, 2), (50, 100, 6, 64, 1), (37, 128, 4, 128, 4),
          (7, 128, 6, 64, 3), (200, 128, 3, 128, 3), (6, 100, 8, 128, 2)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b%d_L%d_H%d_N%d_G%d" % s)
def test_onetile_every_output(ssd, shape):
    batch, L, H, N, G = shape
    inp = si.bidir_inputs(batch, L, H, 64, N, G, "bf16", seed=batch + L + G, device="cuda")
    o = full_oracle(inp)
    for rep in range(2):     # twice on the same workspace and output buffer
        y = run(ssd, inp)
        check(to_f64(y), o, torch.bfloat16, f"one-tile {shape} call {rep}")


def test_onetile_decay_range(ssd):
    """Per-head decays from mild to extreme: the decay span of a 32-token
    block runs from below 1 to thousands, so the diagonal mask blocks take both
    their factorised form and the per-entry exponential."""
    inp = si.bidir_inputs(40, 128, 4, 64, 128, 1, "bf16", seed=11, device="cuda")
    inp["A"] = -torch.tensor([[1.0, 50.0, 300.0, 3000.0], [2.0, 80.0, 500.0, 2000.0]], device="cuda")
    inp["dt"] = (inp["dt"].float() * 3).clamp(max=0.1).to(torch.bfloat16).contiguous()
    check(to_f64(run(ssd, inp)), full_oracle(inp), torch.bfloat16, "one-tile decay range")


def test_onetile_matches_other_tensor_core_path(ssd):
    """Same inputs through the one-tile and the fused kernels: both within the
    bar of the oracle, and close to each other."""
    inp = si.bidir_inputs(30, 128, 8, 64, 128, 2, "bf16", seed=3, device="cuda")
    y1 = run(ssd, inp)
    y2 = ssd.ssd_bidir_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], path=ssd.SSD_PATH_FUSED)
    torch.cuda.synchronize()
    o = full_oracle(inp)
    check(to_f64(y1), o, torch.bfloat16, "one-tile")
    check(to_f64(y2), o, torch.bfloat16, "fused")


def test_onetile_full_size_sampled(ssd):
    """The packed 128-token workload (512 sequences x 24 heads, B/C shared by
    all heads) in one launch, sampled units against the oracle."""
    w = si.WORKLOADS["packed128_b512_g1"]
    inp = si.workload_inputs(w, device="cuda")
    out = run(ssd, inp)
    units = sample_units(w.batch, w.nheads, 16, seed=9)
    for (b, h), o in oracle_units(inp, units).items():
        check(to_f64(out[b, :, h]), o, torch.bfloat16, f"packed128 unit {(b, h)}")


def test_onetile_rejects_longer_sequences(ssd):
    inp = si.bidir_inputs(1, 129, 2, 64, 128, 1, "bf16", seed=1, device="cuda")
    with pytest.raises(ssd.SSDError) as e:
        run(ssd, inp)
    assert e.value.status == ssd.SSD_ERR_UNSUPPORTED
