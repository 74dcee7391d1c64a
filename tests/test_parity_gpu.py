"""GPU parity: the library's kernels against the fp64 oracle, element by element,
on the same seeded inputs. Tolerances are in paritylib (1e-4 relative for fp32
I/O, 2e-2 of output RMS for bf16 I/O)."""
import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as si
from paritylib import check, oracle_units, sample_units, unit_problem
from ssd_inputs import to_f64

pytestmark = pytest.mark.gpu

PATHS = {"simt": 1, "chunked": 2, "fused": 3}
PATHS_ALL = {"auto": 0, **PATHS}
BIDIR_PATHS = {**PATHS, "segmented": 4, "pair": 5}


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_b200 as m
    return m


def run_bidir(ssd, inp, chunk, path):
    out = ssd.ssd_bidir_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                            chunk=chunk, path=path)
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    return to_f64(out)


def full_oracle(inp):
    return oracle.bidir(to_f64(inp["x"]), to_f64(inp["dt"]), to_f64(inp["A"]), to_f64(inp["B"]),
                        to_f64(inp["C"]), to_f64(inp["D"]))


def test_tiny_fp32_L128(ssd):
    w = si.WORKLOADS["tiny_fp32_L128"]
    inp = si.workload_inputs(w, device="cuda")
    y = run_bidir(ssd, inp, w.chunk, 0)
    check(y, full_oracle(inp), torch.float32, w.name)


# (batch, L, H, N, G, chunk): several 128-token tiles, ragged tails, shared and per-head B/C
SMALL = [
    (2, 384, 4, 128, 4, 128),
    (2, 512, 4, 128, 1, 256),
    (3, 200, 6, 64, 2, 64),
    (1, 129, 2, 128, 2, 64),
    (2, 128, 4, 128, 1, 64),
    (1, 1, 2, 64, 1, 64),
    (2, 1000, 3, 128, 3, 256),
]


@pytest.mark.parametrize("path", list(BIDIR_PATHS))
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "b%d_L%d_H%d_N%d_G%d_Q%d" % s)
def test_bf16_small(ssd, shape, path):
    batch, L, H, N, G, chunk = shape
    inp = si.bidir_inputs(batch, L, H, 64, N, G, "bf16", seed=L + H, device="cuda")
    try:
        y = run_bidir(ssd, inp, chunk, BIDIR_PATHS[path])
    except ssd.SSDError as e:
        if e.status == ssd.SSD_ERR_UNSUPPORTED and path != "simt":
            pytest.skip(f"{path} path not available for this shape")
        raise
    check(y, full_oracle(inp), torch.bfloat16, f"{path} {shape}")


@pytest.mark.parametrize("path", list(BIDIR_PATHS))
def test_bf16_decay_range(ssd, path):
    """Per-head decays from mild to extreme (|A| 1 ... 3000, larger dt): the
    decay span of a 32-token block runs from below 1 to thousands, so the
    diagonal mask blocks take both their factorised form and the per-entry
    exponential beyond it. 160 (batch, head) units: every path runs it."""
    inp = si.bidir_inputs(40, 256, 4, 64, 128, 4, "bf16", seed=11, device="cuda")
    inp["A"] = -torch.tensor([[1.0, 50.0, 300.0, 3000.0], [2.0, 80.0, 500.0, 2000.0]], device="cuda")
    inp["dt"] = (inp["dt"].float() * 3).clamp(max=0.1).to(torch.bfloat16).contiguous()
    y = run_bidir(ssd, inp, 128, BIDIR_PATHS[path])
    check(y, full_oracle(inp), torch.bfloat16, f"{path} decay range")


@pytest.mark.parametrize("shape", [(2, 300, 4, 128, 2), (1, 64, 3, 64, 3)])
def test_fp32_small(ssd, shape):
    batch, L, H, N, G = shape
    inp = si.bidir_inputs(batch, L, H, 64, N, G, "f32", seed=7, device="cuda")
    y = run_bidir(ssd, inp, 64, 0)
    check(y, full_oracle(inp), torch.float32, f"fp32 {shape}")


def test_empty_inputs(ssd):
    for batch, L in [(0, 128), (2, 0)]:
        inp = si.bidir_inputs(batch, L, 4, 64, 128, 4, "bf16", device="cuda")
        out = ssd.ssd_bidir_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"])
        assert out.shape == inp["x"].shape


@pytest.mark.parametrize("name,k", [("mixer130m_b32_L1024", 12), ("mixer130m_b32_L1024_g1", 8),
                                    ("packed128_b512_g1", 12), ("long_L65536", 3)])
def test_full_size_sampled(ssd, name, k):
    """Full-size workloads, in the launch configuration the benchmark times,
    checked on a sample of (batch, head) units the oracle computes one by one."""
    w = si.WORKLOADS[name]
    inp = si.workload_inputs(w, device="cuda")
    out = ssd.ssd_bidir_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], chunk=w.chunk)
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    units = sample_units(w.batch, w.nheads, k)
    ref = oracle_units(inp, units)
    for (b, h), o in ref.items():
        check(to_f64(out[b, :, h]), o, torch.bfloat16, f"{name} unit {(b, h)}")


@pytest.mark.parametrize("name,k", [("mixer130m_b32_L1024", 12), ("mixer130m_b32_L1024_g1", 6)])
def test_full_size_sampled_fused(ssd, name, k):
    """The one-CTA fused kernel at the 130M shape (the automatic choice there
    is the two-CTA kernel, tested above), sampled units against the oracle."""
    w = si.WORKLOADS[name]
    inp = si.workload_inputs(w, device="cuda")
    out = ssd.ssd_bidir_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], chunk=w.chunk,
                            path=BIDIR_PATHS["fused"])
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    units = sample_units(w.batch, w.nheads, k, seed=5)
    ref = oracle_units(inp, units)
    for (b, h), o in ref.items():
        check(to_f64(out[b, :, h]), o, torch.bfloat16, f"fused {name} unit {(b, h)}")


@pytest.mark.parametrize("shape", [(3, 256, 2, 128, 2), (1, 1000, 200, 64, 4), (5, 640, 37, 128, 37)],
                         ids=["two_tiles", "many_units_ragged", "odd_tiles"])
def test_pair_every_output(ssd, shape):
    """The two-CTA kernel over whole problems: two tiles (each direction first
    on one), more units than clusters with a ragged last tile, and an odd tile
    count (the middle tile's partial comes from the forward direction); every
    output against the oracle, twice in a row on the same workspace (the
    flags of the first call must not satisfy the second)."""
    batch, L, H, N, G = shape
    inp = si.bidir_inputs(batch, L, H, 64, N, G, "bf16", seed=L + H, device="cuda")
    o = full_oracle(inp)
    for rep in range(2):
        y = run_bidir(ssd, inp, 128, BIDIR_PATHS["pair"])
        check(y, o, torch.bfloat16, f"pair {shape} call {rep}")


@pytest.mark.parametrize("shape", [(64, 128, 8, 128, 2), (50, 100, 6, 64, 1), (37, 128, 4, 128, 4)],
                         ids=["L128_G2", "L100_G1_ragged", "L128_G4_no_sharing"])
def test_one_tile_sequences_sharing_c_b(ssd, shape):
    """Hundreds of one-tile sequences: each CTA takes a contiguous range of
    (batch, head) units and reuses the C/B tiles in its ring for consecutive
    heads of one batch element and B/C group (G < H); runs break at batch and
    group boundaries and at the ends of each CTA's range. Every output checked."""
    batch, L, H, N, G = shape
    inp = si.bidir_inputs(batch, L, H, 64, N, G, "bf16", seed=batch + G, device="cuda")
    y = run_bidir(ssd, inp, 64, PATHS["fused"])
    check(y, full_oracle(inp), torch.bfloat16, f"one-tile {shape}")


def _oracle_of(inp):
    return oracle.bidir(*(to_f64(inp[k]) for k in ("x", "dt", "A", "B", "C", "D")))


def test_flip_identity_gpu(ssd):
    """The reverse scan equals the forward scan run on the flipped sequence,
    each direction checked on its own against the oracle (adding two
    separately rounded bf16 outputs would double the rounding)."""
    inp = si.bidir_inputs(2, 512, 4, 64, 128, 4, "bf16", seed=3, device="cuda")
    run = lambda d: to_f64(ssd.ssd_bidir_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], chunk=128))
    check(run(inp), _oracle_of(inp), torch.bfloat16, "both directions")
    # forward alone: reverse C and D zeroed
    fwd = dict(inp, C=inp["C"].clone(), D=inp["D"].clone())
    fwd["C"][1] = 0
    fwd["D"][1] = 0
    check(run(fwd), _oracle_of(fwd), torch.bfloat16, "forward alone")
    # reverse alone, as the reference the flipped run must reproduce
    rev = dict(inp, C=inp["C"].clone(), D=inp["D"].clone())
    rev["C"][0] = 0
    rev["D"][0] = 0
    o_rev = _oracle_of(rev)
    # the reverse direction's parameters, flipped, run as the forward scan
    flip1 = lambda t: torch.flip(t, dims=[1])
    fl = dict(x=flip1(inp["x"]).contiguous(),
              dt=torch.stack([flip1(inp["dt"][1]), torch.zeros_like(inp["dt"][1])]).contiguous(),
              A=torch.stack([inp["A"][1], inp["A"][1]]).contiguous(),
              B=torch.stack([flip1(inp["B"][1]), torch.zeros_like(inp["B"][1])]).contiguous(),
              C=torch.stack([flip1(inp["C"][1]), torch.zeros_like(inp["C"][1])]).contiguous(),
              D=torch.stack([inp["D"][1], torch.zeros_like(inp["D"][1])]).contiguous())
    check(np.flip(run(fl), axis=1), o_rev, torch.bfloat16, "flipped forward = reverse")


@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_chunk_invariance(ssd, chunk):
    inp = si.bidir_inputs(2, 768, 4, 64, 128, 4, "bf16", seed=11, device="cuda")
    y = run_bidir(ssd, inp, chunk, 0)
    y128 = run_bidir(ssd, inp, 128, 0)
    o = full_oracle(inp)
    check(y, o, torch.bfloat16, f"chunk {chunk}")
    # both within 2e-2 rms (plus half an ulp each) of the oracle, so within
    # 4e-2 rms plus one ulp of each other
    from paritylib import half_ulp_bf16, rms
    d = np.abs(y - y128) - 2 * half_ulp_bf16(np.maximum(np.abs(y), np.abs(y128)))
    assert np.max(d) <= 4e-2 * rms(o)


# ---------------------------------------------------------------- prefix state

def _paths_for(dtype):
    return ["auto", "simt"] if dtype == "f32" else ["auto", "simt", "chunked", "fused"]


@pytest.mark.parametrize("dtype,path", [(d, p) for d in ("f32", "bf16") for p in _paths_for(d)])
@pytest.mark.parametrize("L,N,G", [(1000, 128, 4), (256, 64, 1), (2000, 64, 2), (1, 128, 4), (0, 128, 4)])
def test_prefix_state(ssd, dtype, path, L, N, G):
    """Every path, with and without a start state; 8 and 16 tiles wrap the
    fused kernel's 5 (N 128) and 3 (N 64) x slots of its state-only mode."""
    inp = si.bidir_inputs(2, L, 4, 64, N, G, dtype, seed=5, device="cuda")
    init = torch.randn(2, 4, 64, N, device="cuda") * 0.5
    for start in (None, init):
        st = ssd.ssd_prefix_state(inp["x"], inp["dt"][0], inp["A"][0], inp["B"][0], init=start, chunk=128,
                                  path=PATHS_ALL[path])
        o = oracle.prefix_state(to_f64(inp["x"]), to_f64(inp["dt"][0]), to_f64(inp["A"][0]),
                                to_f64(inp["B"][0]), init=None if start is None else to_f64(start))
        check(to_f64(st), o, torch.float32 if dtype == "f32" else torch.bfloat16, f"prefix L={L}", state=True)


@pytest.mark.parametrize("path", ["chunked", "fused"])
def test_prefix_state_composes_in_place(ssd, path):
    inp = si.bidir_inputs(2, 640, 4, 64, 128, 4, "bf16", seed=9, device="cuda")
    k = 384
    x, dt, A, B = inp["x"], inp["dt"][0], inp["A"][0], inp["B"][0]
    pid = PATHS[path]
    full = ssd.ssd_prefix_state(x, dt, A, B, path=pid)
    st = ssd.ssd_prefix_state(x[:, :k].contiguous(), dt[:, :k].contiguous(), A, B[:, :k].contiguous(), path=pid)
    ssd.ssd_prefix_state(x[:, k:].contiguous(), dt[:, k:].contiguous(), A, B[:, k:].contiguous(),
                         init=st, out=st, path=pid)  # committing a block in place
    o = oracle.prefix_state(to_f64(x), to_f64(dt), to_f64(A), to_f64(B))
    check(to_f64(st), o, torch.bfloat16, "composed", state=True)
    check(to_f64(full), o, torch.bfloat16, "direct", state=True)


@pytest.mark.parametrize("path", ["chunked", "fused"])
def test_prefix_state_and_block_step_many_units(ssd, path):
    """160 (batch, head) units: more than there are SMs, so the fused kernel's
    CTAs take two units each and carry their barrier phases across them."""
    batch, H, N, G = 40, 4, 128, 2
    data = si.blockstep_inputs(batch, 700, 64, 1, H, 64, N, G, "bf16", seed=13, device="cuda")
    pid = PATHS[path]
    st = ssd.ssd_prefix_state(data["x_pre"], data["dt_pre"], data["A"][0], data["B_pre"], path=pid)
    step = data["steps"][0]
    y = ssd.ssd_block_step(step["x"], step["dt"], data["A"], step["B"], step["C"], data["D"], st, path=pid)
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    st_o = oracle.prefix_state(to_f64(data["x_pre"]), to_f64(data["dt_pre"]), to_f64(data["A"][0]),
                               to_f64(data["B_pre"]))
    check(to_f64(st), st_o, torch.bfloat16, f"{path} prefix, 160 units", state=True)
    check(to_f64(y), _block_oracle(step, data["A"], data["D"], st_o), torch.bfloat16, f"{path} block step, 160 units")


def test_prefix_state_full_size_sampled(ssd):
    """The 262144-token prefix of the block-diffusion workload, sampled units."""
    w = si.WORKLOADS["blockstep_prefix262144_blk64"]
    data = si.blockstep_inputs(w.batch, w.seqlen, w.block, 1, w.nheads, w.headdim, w.dstate,
                               w.ngroups, w.dtype, device="cuda")
    st = ssd.ssd_prefix_state(data["x_pre"], data["dt_pre"], data["A"][0], data["B_pre"], chunk=w.chunk)
    torch.cuda.synchronize()
    for b, h in sample_units(w.batch, w.nheads, 3, seed=1):
        g = h // (w.nheads // w.ngroups)
        o = oracle.prefix_state(to_f64(data["x_pre"][b:b + 1, :, h:h + 1]),
                                to_f64(data["dt_pre"][b:b + 1, :, h:h + 1]),
                                to_f64(data["A"][0, h:h + 1]),
                                to_f64(data["B_pre"][b:b + 1, :, g:g + 1]))
        check(to_f64(st[b:b + 1, h:h + 1]), o, torch.bfloat16, f"prefix262144 unit {(b, h)}", state=True)


# ---------------------------------------------------------------- block step

def _block_oracle(step, A, D, state):
    return oracle.block_step(to_f64(step["x"]), to_f64(step["dt"]), to_f64(A), to_f64(step["B"]),
                             to_f64(step["C"]), to_f64(D), state)


@pytest.mark.parametrize("dtype,path", [(d, p) for d in ("f32", "bf16") for p in _paths_for(d)])
@pytest.mark.parametrize("blk,N", [(64, 128), (200, 64)])
def test_block_step_against_oracle(ssd, dtype, path, blk, N):
    data = si.blockstep_inputs(2, 1000, blk, 3, 4, 64, N, 2, dtype, device="cuda")
    st = ssd.ssd_prefix_state(data["x_pre"], data["dt_pre"], data["A"][0], data["B_pre"])
    st_o = oracle.prefix_state(to_f64(data["x_pre"]), to_f64(data["dt_pre"]), to_f64(data["A"][0]),
                               to_f64(data["B_pre"]))
    io = torch.float32 if dtype == "f32" else torch.bfloat16
    for k, step in enumerate(data["steps"]):
        y = ssd.ssd_block_step(step["x"], step["dt"], data["A"], step["B"], step["C"], data["D"], st,
                               path=PATHS_ALL[path])
        check(to_f64(y), _block_oracle(step, data["A"], data["D"], st_o), io, f"{path} step {k}")
    # no prefix state: the forward scan starts from zero
    step = data["steps"][0]
    y = ssd.ssd_block_step(step["x"], step["dt"], data["A"], step["B"], step["C"], data["D"], None,
                           path=PATHS_ALL[path])
    check(to_f64(y), _block_oracle(step, data["A"], data["D"], None), io, f"{path} step from zero")


def test_block_steps_leave_prefix_state_untouched(ssd):
    """32 denoising steps read the cached state and never write it."""
    w = si.WORKLOADS["blockstep_prefix262144_blk64"]
    data = si.blockstep_inputs(w.batch, 4096, w.block, w.steps, w.nheads, 64, w.dstate, w.ngroups,
                               "bf16", device="cuda")
    st = ssd.ssd_prefix_state(data["x_pre"], data["dt_pre"], data["A"][0], data["B_pre"])
    before = st.clone()
    outs = []
    for step in data["steps"]:
        outs.append(ssd.ssd_block_step(step["x"], step["dt"], data["A"], step["B"], step["C"],
                                       data["D"], st))
    torch.cuda.synchronize()
    assert torch.equal(st, before)
    # spot-check the first and last step against the oracle from the oracle's own state
    st_o = oracle.prefix_state(to_f64(data["x_pre"]), to_f64(data["dt_pre"]), to_f64(data["A"][0]),
                               to_f64(data["B_pre"]))
    for k in (0, w.steps - 1):
        check(to_f64(outs[k]), _block_oracle(data["steps"][k], data["A"], data["D"], st_o),
              torch.bfloat16, f"step {k}")


def test_block_step_forward_part_matches_full_scan(ssd):
    """Forward part of a block step = last T outputs of the forward scan over
    prefix ++ block; reverse part = the reverse scan over the block alone."""
    inp = si.bidir_inputs(2, 512 + 64, 4, 64, 128, 4, "bf16", seed=21, device="cuda")
    k = 512
    x, dt, A, B, C, D = (inp[n] for n in ("x", "dt", "A", "B", "C", "D"))
    st = ssd.ssd_prefix_state(x[:, :k].contiguous(), dt[0, :, :k].contiguous(), A[0], B[0, :, :k].contiguous())
    sl = lambda t: t[:, :, k:].contiguous()
    y = to_f64(ssd.ssd_block_step(x[:, k:].contiguous(), sl(dt), A, sl(B), sl(C), D, st))
    Cf = C.clone(); Cf[1] = 0
    Dz = torch.zeros_like(D)
    y_fwd = to_f64(ssd.ssd_bidir_fwd(x, dt, A, B, Cf, Dz, chunk=128))[:, k:]
    Cr = sl(C).clone(); Cr[0] = 0
    y_rev = to_f64(ssd.ssd_bidir_fwd(x[:, k:].contiguous(), sl(dt), A, sl(B), Cr, D, chunk=64))
    ref = oracle.block_step(to_f64(x[:, k:]), to_f64(sl(dt)), to_f64(A), to_f64(sl(B)), to_f64(sl(C)),
                            to_f64(D), oracle.prefix_state(to_f64(x[:, :k]), to_f64(dt[0, :, :k]),
                                                           to_f64(A[0]), to_f64(B[0, :, :k])))
    check(y, ref, torch.bfloat16, "block step")
    # each part on its own (adding two rounded bf16 outputs would double the rounding)
    xk = to_f64(x[:, k:])
    pre = oracle.prefix_state(to_f64(x[:, :k]), to_f64(dt[0, :, :k]), to_f64(A[0]), to_f64(B[0, :, :k]))
    ref_f = oracle.block_step(xk, to_f64(sl(dt)), to_f64(A), to_f64(sl(B)), to_f64(sl(Cf)),
                              np.zeros((2, 4)), pre)
    ref_r = oracle.block_step(xk, to_f64(sl(dt)), to_f64(A), to_f64(sl(B)), to_f64(Cr),
                              to_f64(D), None)
    check(y_fwd, ref_f, torch.bfloat16, "forward scan over prefix ++ block, last T")
    check(y_rev, ref_r, torch.bfloat16, "reverse scan over the block alone")
