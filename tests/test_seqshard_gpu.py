"""GPU parity of the segment entry points and of the sequence-sharded mixer
run on one GPU: the segments a process group would hold are processed one
after the other in one process, their states stacked segment-major exactly
as the all_gather of seqshard.py stacks them. Everything is compared with
the fp64 oracle over the whole sequence (tolerances in paritylib)."""
import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as si
from paritylib import check
from ssd_inputs import to_f64

pytestmark = pytest.mark.gpu

# (batch, L, H, N, G): ragged tails, shared and per-head B/C, 8 to 160 units;
# the last one has too few units to fill the GPU, so both calls split each
# sequence into 16 segments of 1024 tokens internally
SHAPES = [(2, 300, 4, 128, 2), (4, 384, 24, 64, 24), (40, 256, 4, 128, 4), (1, 1, 2, 64, 1),
          (1, 16384, 8, 128, 8)]


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_b200 as m
    return m


def _flip(a):
    return np.flip(a, axis=1).copy()


def _f64(inp, *names):
    return [to_f64(inp[n]) for n in names]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b%d_L%d_H%d_N%d_G%d" % s)
def test_segment_states_against_oracle(ssd, shape):
    batch, L, H, N, G = shape
    inp = si.bidir_inputs(batch, L, H, 64, N, G, "bf16", seed=L + 3, device="cuda")
    fs, fd, rs, rd = ssd.ssd_segment_states(inp["x"], inp["dt"], inp["A"], inp["B"])
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    x, dt, A, B = _f64(inp, "x", "dt", "A", "B")
    check(to_f64(fs), oracle.prefix_state(x, dt[0], A[0], B[0]), torch.bfloat16, "forward state", state=True)
    # the reverse state before the first token: a forward scan of the flipped sequence
    check(to_f64(rs), oracle.prefix_state(_flip(x), _flip(dt[1]), A[1], _flip(B[1])), torch.bfloat16,
          "reverse state", state=True)
    check(to_f64(fd), np.exp(A[0][None, :] * dt[0].sum(axis=1)), torch.float32, "forward decay")
    check(to_f64(rd), np.exp(A[1][None, :] * dt[1].sum(axis=1)), torch.float32, "reverse decay")


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b%d_L%d_H%d_N%d_G%d" % s)
def test_bidir_seeded_against_oracle(ssd, shape):
    batch, L, H, N, G = shape
    inp = si.bidir_inputs(batch, L, H, 64, N, G, "bf16", seed=L + 4, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(L)
    fi = torch.randn(batch, H, 64, N, device="cuda", generator=gen) * 0.5
    ri = torch.randn(batch, H, 64, N, device="cuda", generator=gen) * 0.5
    args = [inp[n] for n in ("x", "dt", "A", "B", "C", "D")]
    o64 = _f64(inp, "x", "dt", "A", "B", "C", "D")
    for f, r in ((fi, ri), (None, ri), (fi, None), (None, None)):
        y = ssd.ssd_bidir_fwd_seeded(*args, f, r)
        torch.cuda.synchronize()
        assert ssd.ssd_get_device_status() == 0
        o = oracle.bidir_seeded(*o64, None if f is None else to_f64(f), None if r is None else to_f64(r))
        check(to_f64(y), o, torch.bfloat16, f"seeded fwd={f is not None} rev={r is not None}")


def _sharded_one_gpu(ssd, inp, nseg):
    """What seqshard.ssd_bidir_fwd_seq_sharded computes on nseg ranks, run here
    segment after segment on one GPU."""
    L = inp["x"].shape[1]
    ls = L // nseg
    seg = lambda t, axis, s: t.narrow(axis, s * ls, ls).contiguous()
    parts = []
    for s in range(nseg):
        parts.append(dict(x=seg(inp["x"], 1, s), dt=seg(inp["dt"], 2, s), B=seg(inp["B"], 2, s),
                          C=seg(inp["C"], 2, s)))
    states = [ssd.ssd_segment_states(p["x"], p["dt"], inp["A"], p["B"]) for p in parts]
    gathered = [torch.stack([st[k] for st in states]) for k in range(4)]
    outs, carried = [], []
    for s, p in enumerate(parts):
        fi, ri = ssd.ssd_segment_carry(*gathered, s)
        carried.append((fi, ri))
        outs.append(ssd.ssd_bidir_fwd_seeded(p["x"], p["dt"], inp["A"], p["B"], p["C"], inp["D"], fi, ri))
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    return torch.cat(outs, dim=1), carried


@pytest.mark.parametrize("nseg,shape", [(3, (2, 900, 4, 128, 4)), (4, (3, 1024, 8, 64, 2)), (2, (1, 256, 32, 128, 32)),
                                        (2, (1, 32768, 8, 128, 8))],
                         ids=["3seg_L900", "4seg_L1024_G2", "2seg_H32", "2seg_L32768_few_units"])
def test_sequence_sharded_matches_whole_sequence(ssd, nseg, shape):
    batch, L, H, N, G = shape
    inp = si.bidir_inputs(batch, L, H, 64, N, G, "bf16", seed=L + nseg, device="cuda")
    y, carried = _sharded_one_gpu(ssd, inp, nseg)
    x, dt, A, B, C, D = _f64(inp, "x", "dt", "A", "B", "C", "D")
    check(to_f64(y), oracle.bidir(x, dt, A, B, C, D), torch.bfloat16, f"{nseg} segments")
    # the carried states are the states the rest of the sequence leaves
    ls = L // nseg
    for s, (fi, ri) in enumerate(carried):
        t0, t1 = s * ls, (s + 1) * ls
        if t0 > 0:
            check(to_f64(fi), oracle.prefix_state(x[:, :t0], dt[0][:, :t0], A[0], B[0][:, :t0]), torch.bfloat16,
                  f"state into segment {s}", state=True)
        else:
            assert torch.count_nonzero(fi) == 0
        if t1 < L:
            check(to_f64(ri), oracle.prefix_state(_flip(x[:, t1:]), _flip(dt[1][:, t1:]), A[1], _flip(B[1][:, t1:])),
                  torch.bfloat16, f"reverse state into segment {s}", state=True)
        else:
            assert torch.count_nonzero(ri) == 0
