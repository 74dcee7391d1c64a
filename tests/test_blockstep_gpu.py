"""GPU parity of the one-tile block-step kernel (ssd_block_step with
SSD_PATH_BLOCK, the automatic choice for bf16 blocks of at most 64 tokens)
against the fp64 oracle's block step (oracle.block_step), element by element.

The cached prefix state handed to the kernel is the oracle's own state
rounded to fp32, so the comparison isolates the block step. Shapes cover a
full 64-token block, ragged blocks (50, 33 and 1 tokens), d_state 64 and
128, B/C shared by groups of heads and per head, no prefix state, more
(batch, head) units than SMs, and the block-diffusion workload's shape
(4 x 32 heads, d_state 128). Tolerance: paritylib's bf16 bar.
"""
import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as si
from paritylib import check
from ssd_inputs import to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_b200 as m
    return m


# (batch, T, H, N, G, with prefix state)
SHAPES = [(2, 64, 4, 128, 2, True), (3, 50, 6, 64, 3, True), (1, 1, 2, 128, 1, True), (2, 33, 4, 128, 4, False),
          (40, 64, 4, 128, 2, True), (4, 64, 32, 128, 32, True)]


def _ids(s):
    return "b%d_T%d_H%d_N%d_G%d_%s" % (s[:5] + ("prefix" if s[5] else "zero",))


@pytest.mark.parametrize("shape", SHAPES, ids=_ids)
def test_block_kernel_against_oracle(ssd, shape):
    batch, T, H, N, G, with_prefix = shape
    data = si.blockstep_inputs(batch, 96, T, 2, H, 64, N, G, "bf16", seed=T + H, device="cuda")
    st_o = None
    st = None
    if with_prefix:
        st_o = oracle.prefix_state(to_f64(data["x_pre"]), to_f64(data["dt_pre"]), to_f64(data["A"][0]),
                                   to_f64(data["B_pre"]))
        st = torch.from_numpy(st_o.astype(np.float32)).to("cuda")
        st_o = st_o.astype(np.float32).astype(np.float64)
    for k, step in enumerate(data["steps"]):
        y = ssd.ssd_block_step(step["x"], step["dt"], data["A"], step["B"], step["C"], data["D"], st,
                               path=ssd.SSD_PATH_BLOCK)
        y_auto = ssd.ssd_block_step(step["x"], step["dt"], data["A"], step["B"], step["C"], data["D"], st)
        torch.cuda.synchronize()
        assert ssd.ssd_get_device_status() == 0
        assert torch.equal(y, y_auto), "the automatic choice runs the one-tile kernel"
        o = oracle.block_step(to_f64(step["x"]), to_f64(step["dt"]), to_f64(data["A"]), to_f64(step["B"]),
                              to_f64(step["C"]), to_f64(data["D"]), st_o)
        check(to_f64(y), o, torch.bfloat16, f"block kernel {shape} step {k}")


def test_block_kernel_leaves_state_untouched(ssd):
    data = si.blockstep_inputs(2, 96, 64, 1, 4, 64, 128, 2, "bf16", seed=5, device="cuda")
    st = ssd.ssd_prefix_state(data["x_pre"], data["dt_pre"], data["A"][0], data["B_pre"])
    before = st.clone()
    step = data["steps"][0]
    ssd.ssd_block_step(step["x"], step["dt"], data["A"], step["B"], step["C"], data["D"], st,
                       path=ssd.SSD_PATH_BLOCK)
    torch.cuda.synchronize()
    assert torch.equal(st, before)


def test_block_kernel_rejects_long_blocks(ssd):
    data = si.blockstep_inputs(1, 96, 65, 1, 2, 64, 128, 1, "bf16", seed=6, device="cuda")
    step = data["steps"][0]
    with pytest.raises(RuntimeError):
        ssd.ssd_block_step(step["x"], step["dt"], data["A"], step["B"], step["C"], data["D"], None,
                           path=ssd.SSD_PATH_BLOCK)
