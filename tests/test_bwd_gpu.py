"""GPU parity of the backward pass (ssd_bidir_bwd) against the fp64 oracle's
gradients (oracle.bidir_bwd, pinned in test_oracle_bwd_pins.py), element by
element on the same seeded inputs.

Gradients are fp32 results computed in fp32 from the same (rounded) inputs the
oracle sees, whatever the I/O dtype, so every gradient is held to the fp32
bar of paritylib: max |g - o| / max(|o|, rms(o)) <= 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as si
from paritylib import TOL_F32, err_f32, sample_units
from ssd_inputs import to_f64

pytestmark = pytest.mark.gpu

NAMES = ("x", "dt", "A", "B", "C", "D")
GRADS = ("dx", "ddt", "dA", "dB", "dC", "dD")


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_b200 as m
    return m


def _dy(shape, io, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn(shape, generator=g, device="cuda").to(io).contiguous()


def _check_all(g, o, what):
    errs = {}
    for k in GRADS:
        y = to_f64(g[k])
        assert np.isfinite(y).all(), f"{what} {k}: non-finite"
        errs[k] = err_f32(y, o[k])
        assert errs[k] <= TOL_F32, f"{what} {k}: max rel err {errs[k]:.3e} > {TOL_F32}"
    return errs


# (batch, L, H, N, G, io): ragged lengths across the 32-token staging, G < H
# and G = H, both d_state values, both I/O dtypes, a single token
SHAPES = [(2, 100, 4, 128, 2, "f32"), (1, 300, 2, 64, 2, "bf16"), (2, 64, 3, 128, 3, "bf16"),
          (1, 1, 2, 64, 1, "f32"), (3, 257, 4, 128, 4, "bf16"), (2, 33, 6, 64, 3, "f32")]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b%d_L%d_H%d_N%d_G%d_%s" % s)
def test_bwd_against_oracle(ssd, shape):
    batch, L, H, N, G, io = shape
    inp = si.bidir_inputs(batch, L, H, 64, N, G, io, seed=L + H, device="cuda")
    dy = _dy(inp["x"].shape, inp["x"].dtype, seed=L)
    g = ssd.ssd_bidir_bwd(*(inp[k] for k in NAMES), dy)
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    o = oracle.bidir_bwd(*(to_f64(inp[k]) for k in NAMES), to_f64(dy))
    _check_all(g, o, f"bwd {shape}")


def test_bwd_is_deterministic_with_per_head_groups(ssd):
    """G = H: every output element has a fixed order of additions."""
    inp = si.bidir_inputs(2, 200, 4, 64, 128, 4, "bf16", seed=9, device="cuda")
    dy = _dy(inp["x"].shape, inp["x"].dtype, seed=10)
    g1 = ssd.ssd_bidir_bwd(*(inp[k] for k in NAMES), dy)
    g2 = ssd.ssd_bidir_bwd(*(inp[k] for k in NAMES), dy)
    torch.cuda.synchronize()
    for k in ("dx", "ddt", "dB", "dC"):
        assert torch.equal(g1[k], g2[k]), k


def test_bwd_empty(ssd):
    inp = si.bidir_inputs(2, 0, 4, 64, 128, 4, "bf16", device="cuda")
    dy = torch.empty_like(inp["x"])
    g = ssd.ssd_bidir_bwd(*(inp[k] for k in NAMES), dy)
    torch.cuda.synchronize()
    assert float(g["dA"].abs().sum()) == 0.0 and float(g["dD"].abs().sum()) == 0.0


def test_bwd_full_size_130m(ssd):
    """The 130M mixer shape (32 x 1024 tokens, 24 heads, d_state 128, bf16):
    per-unit gradients on sampled (batch, head) units, and dA, dD (sums over
    the batch) against the oracle over every unit."""
    w = si.WORKLOADS["mixer130m_b32_L1024"]
    inp = si.workload_inputs(w, device="cuda")
    dy = _dy(inp["x"].shape, inp["x"].dtype, seed=77)
    g = ssd.ssd_bidir_bwd(*(inp[k] for k in NAMES), dy)
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    o = oracle.bidir_bwd(*(to_f64(inp[k]) for k in NAMES), to_f64(dy))
    for k in ("dA", "dD"):
        e = err_f32(to_f64(g[k]), o[k])
        assert e <= TOL_F32, f"130M {k}: {e:.3e}"
    for b, h in sample_units(w.batch, w.nheads, 6, seed=3):
        for k, sl in (("dx", np.s_[b, :, h]), ("ddt", np.s_[:, b, :, h]), ("dB", np.s_[:, b, :, h]),
                      ("dC", np.s_[:, b, :, h])):
            e = err_f32(to_f64(g[k])[sl], o[k][sl])
            assert e <= TOL_F32, f"130M {k} unit {(b, h)}: {e:.3e}"


# (batch, L, H, N, G, io): the seeded backward, with start states in both
# directions (ragged length, G < H) and the block step's (a prefix state, no
# reverse start state)
SEEDED = [(2, 100, 4, 128, 2, "f32"), (1, 300, 2, 64, 2, "bf16"), (3, 33, 4, 128, 4, "bf16")]


def _state(batch, H, N, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return (torch.randn(batch, H, 64, N, generator=g, device="cuda") * 0.5).contiguous()


@pytest.mark.parametrize("shape", SEEDED, ids=lambda s: "b%d_L%d_H%d_N%d_G%d_%s" % s)
def test_seeded_bwd_against_oracle(ssd, shape):
    batch, L, H, N, G, io = shape
    inp = si.bidir_inputs(batch, L, H, 64, N, G, io, seed=L + 2 * H, device="cuda")
    dy = _dy(inp["x"].shape, inp["x"].dtype, seed=L + 1)
    pre, suf = _state(batch, H, N, 11), _state(batch, H, N, 12)
    g = ssd.ssd_bidir_bwd(*(inp[k] for k in NAMES), dy, fwd_init=pre, rev_init=suf)
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    o = oracle.bidir_bwd(*(to_f64(inp[k]) for k in NAMES), to_f64(dy), prefix=to_f64(pre), suffix=to_f64(suf))
    _check_all(g, o, f"seeded bwd {shape}")
    for k, ok in (("d_fwd_init", "dprefix"), ("d_rev_init", "dsuffix")):
        e = err_f32(to_f64(g[k]), o[ok])
        assert e <= TOL_F32, f"seeded bwd {shape} {k}: {e:.3e}"


@pytest.mark.parametrize("shape", [(2, 64, 4, 128, 4), (3, 50, 6, 64, 3)], ids=["T64_N128", "T50_N64_ragged"])
def test_block_step_bwd_against_oracle(ssd, shape):
    """The block step's gradients: forward scan from a cached prefix state,
    reverse scan from zero at the block end."""
    batch, T, H, N, G = shape
    data = si.blockstep_inputs(batch, 96, T, 1, H, 64, N, G, "bf16", seed=T + H, device="cuda")
    pre_o = oracle.prefix_state(to_f64(data["x_pre"]), to_f64(data["dt_pre"]), to_f64(data["A"][0]),
                                to_f64(data["B_pre"]))
    pre = torch.from_numpy(pre_o.astype(np.float32)).to("cuda")
    step = data["steps"][0]
    dy = _dy(step["x"].shape, step["x"].dtype, seed=T)
    g = ssd.ssd_block_step_bwd(step["x"], step["dt"], data["A"], step["B"], step["C"], data["D"], pre, dy)
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    inp = {"x": step["x"], "dt": step["dt"], "A": data["A"], "B": step["B"], "C": step["C"], "D": data["D"]}
    o = oracle.bidir_bwd(*(to_f64(inp[k]) for k in NAMES), to_f64(dy), prefix=to_f64(pre))
    _check_all(g, o, f"block step bwd {shape}")
    e = err_f32(to_f64(g["d_prefix_state"]), o["dprefix"])
    assert e <= TOL_F32, f"block step bwd {shape} d_prefix_state: {e:.3e}"


def test_seeded_bwd_empty(ssd):
    inp = si.bidir_inputs(2, 0, 4, 64, 128, 4, "bf16", device="cuda")
    pre = _state(2, 4, 128, 13)
    g = ssd.ssd_bidir_bwd(*(inp[k] for k in NAMES), torch.empty_like(inp["x"]), fwd_init=pre)
    torch.cuda.synchronize()
    assert float(g["d_fwd_init"].abs().sum()) == 0.0
