"""GPU parity of the mixer's input and output steps against the oracle:
  * ssd_bidir_fwd_x2 (each direction scans its own x) on the two-CTA
    tensor-core kernel and on the sequential scan, against oracle.bidir_x2;
  * ssd_mixer_block_fwd (conv1d + SiLU per direction, dt from the raw
    projection, the mixer, the gated RMS norm) end to end against
    oracle.mixer_block's steps, with the intermediates rounded to the I/O
    dtype where the block stores them (the conv output, dt and the mixer
    output: the layer's activations are kept in the I/O dtype), at the 130M
    shape's channel counts among others.
Tolerances: the mixer alone, paritylib's (fp32 1e-4 relative; bf16 2e-2 of
RMS beyond the final rounding, and 3e-3 RMS error). The block with bf16 I/O
stores the mixer output in bf16 and then normalises each token, which is
invariant to the token's scale: an intermediate rounding of one ulp (2^-8
relative) moves an output element by about that fraction of itself, and the
outputs are heavy tailed (elements up to ~20 rms), so the block's bar is the
same 2e-2 taken relative to each element, floored at the RMS:
max_i (|y_i - o_i| - ulp(y_i)/2) / max(|o_i|, rms(o)) <= 2e-2, plus the RMS
bar 3e-3. fp32 I/O keeps the fp32 bar.
"""
import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as si
from paritylib import TOL_BF16, TOL_BF16_RMS, check, half_ulp_bf16, rms, rms_err
from ssd_inputs import to_f64

pytestmark = pytest.mark.gpu

NAMES = ("dt", "A", "B", "C", "D")


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_b200 as m
    return m


def _rng_tensor(shape, seed, scale=1.0, dtype=torch.float32):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return (torch.randn(shape, generator=g, device="cuda") * scale).to(dtype).contiguous()


# (batch, L, H, N, G, io): two-CTA kernel (bf16, > 1 tile, incl. ragged), the
# sequential scan (one tile, fp32)
X2_SHAPES = [(2, 384, 8, 128, 8, "bf16"), (3, 200, 6, 64, 2, "bf16"), (2, 100, 4, 128, 1, "bf16"),
             (2, 150, 4, 64, 2, "f32"), (1, 257, 2, 128, 2, "f32")]


@pytest.mark.parametrize("shape", X2_SHAPES, ids=lambda s: "b%d_L%d_H%d_N%d_G%d_%s" % s)
def test_bidir_fwd_x2_against_oracle(ssd, shape):
    batch, L, H, N, G, io = shape
    inp = si.bidir_inputs(batch, L, H, 64, N, G, io, seed=L + 3 * H, device="cuda")
    x2 = torch.stack([inp["x"], _rng_tensor(inp["x"].shape, L, dtype=inp["x"].dtype)]).contiguous()
    y = ssd.ssd_bidir_fwd_x2(x2, *(inp[k] for k in NAMES))
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    o = oracle.bidir_x2(to_f64(x2), *(to_f64(inp[k]) for k in NAMES))
    check(to_f64(y), o, inp["x"].dtype, f"x2 {shape}")


def _round(a, io):
    """a rounded to the I/O dtype (round to nearest even), back in fp64."""
    return torch.from_numpy(np.asarray(a)).to(io).to(torch.float64).numpy()


# (batch, L, H, N, G, io, K)
BLOCK_SHAPES = [(2, 300, 8, 128, 8, "bf16", 4), (1, 1024, 24, 128, 24, "bf16", 4), (2, 100, 4, 64, 2, "bf16", 3),
                (2, 129, 4, 64, 2, "f32", 4)]


@pytest.mark.parametrize("shape", BLOCK_SHAPES, ids=lambda s: "b%d_L%d_H%d_N%d_G%d_%s_K%d" % s)
def test_mixer_block_against_oracle(ssd, shape):
    batch, L, H, N, G, iod, K = shape
    io = torch.bfloat16 if iod == "bf16" else torch.float32
    P = 64
    cin = H * P + 2 * G * N
    xbc = _rng_tensor((batch, L, cin), 1, dtype=io)
    z = _rng_tensor((batch, L, H, P), 2, dtype=io)
    dt_raw = _rng_tensor((2, batch, L, H), 3, dtype=io)
    conv_w = _rng_tensor((2, cin, K), 4, scale=0.5)
    conv_b = _rng_tensor((2, cin), 5, scale=0.1)
    dt_bias = (torch.log(torch.expm1(torch.full((2, H), 0.02, device="cuda")))
               + _rng_tensor((2, H), 6, scale=0.3)).contiguous()
    A = -torch.exp(_rng_tensor((2, H), 7, scale=0.5)).contiguous()
    D = _rng_tensor((2, H), 8)
    norm_w = (1.0 + _rng_tensor((H * P,), 9, scale=0.1)).contiguous()
    dt_min, dt_max, eps = 1e-3, 0.1, 1e-5
    out = ssd.ssd_mixer_block_fwd(xbc, z, dt_raw, conv_w, conv_b, dt_bias, A, D, norm_w, H, G, N,
                                  dt_min=dt_min, dt_max=dt_max, norm_eps=eps)
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    # the oracle's steps, rounded where the block stores its intermediates
    u = oracle.conv_silu(to_f64(xbc), to_f64(conv_w), to_f64(conv_b))
    if io == torch.bfloat16:
        u = _round(u, io)
    x2, B, C = oracle.split_xbc(u, H, P, G, N)
    dt = oracle.dt_prep(to_f64(dt_raw), to_f64(dt_bias), dt_min, dt_max)
    if io == torch.bfloat16:
        dt = _round(dt, io)
    y = oracle.bidir_x2(x2, dt, to_f64(A), B, C, to_f64(D))
    if io == torch.bfloat16:
        y = _round(y, io)
    o = oracle.gated_rmsnorm(y, to_f64(z), to_f64(norm_w), eps)
    g = to_f64(out)
    if io == torch.float32:
        check(g, o, io, f"block {shape}")
        return
    assert np.isfinite(g).all()
    d = np.maximum(np.abs(g - o) - half_ulp_bf16(np.maximum(np.abs(g), np.abs(o))), 0.0)
    e = float(np.max(d / np.maximum(np.abs(o), rms(o))))
    r = rms_err(g, o)
    assert e <= TOL_BF16, f"block {shape}: elementwise err {e:.3e} > {TOL_BF16} (rms err {r:.2e})"
    assert r <= TOL_BF16_RMS, f"block {shape}: rms err {r:.3e}"
