"""Seeded synthetic inputs and named workloads for the bidirectional SSD mixer.

This module is shared by the tests, the benchmark and the smoke check, and is
the only thing the CUDA path and the fp64 oracle have in common. It draws
random numbers and casts them to the I/O dtype; it holds none of the mixer's
arithmetic.

Recipe (every workload, seed 0 unless stated):
  x     ~ N(0, 1)                                          (batch, L, H, P)
  for each direction d in (forward, reverse), in this order:
    dt  = clamp(softplus(z - 4), 1e-3, 0.1),  z ~ N(0, 1)  (batch, L, H)
    A   = -exp(u),  u ~ U(log 1, log 16)                   (H,)      fp32
    B   ~ N(0, 1) / 8                                      (batch, L, G, N)
    C   ~ N(0, 1) / 8                                      (batch, L, G, N)
    D   ~ N(0, 1)                                          (H,)      fp32
x, dt, B and C are drawn in fp32 and then rounded (nearest-even) to the I/O
dtype; the rounded values are what both the GPU and the oracle see. The
spread 1/8 = 1/sqrt(64) is kept for d_state 128 too ("same distributions").
Random numbers come from torch.Generator on the device the tensors live on,
so one seed gives different (but fixed) values on CPU and on CUDA.

The shapes follow the workloads the pages describe: a 130M DiffMamba mixer
at L = 1024 (DiffMamba model card, Model details: hidden 768, 12 blocks,
sequence length 1024, headdim 64), LM1B packed to 128 tokens with batch 512,
and the 65K / 262K long-context lengths of the block-diffusion paper
("Training Hybrid Block Diffusion Language Models with Partial
Bidirectionality", Abstract). No text corpus is used: only these shapes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, asdict, replace

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    """One named problem size. For block-step workloads ``seqlen`` is the
    cached prefix length and ``block``/``steps`` describe the active block."""
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk: int
    dtype: str
    block: int = 0
    steps: int = 0

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    def as_dict(self) -> dict:
        return asdict(self)


WORKLOADS = {
    w.name: w
    for w in [
        # parity case: fp32 I/O, one small layer
        Workload("tiny_fp32_L128", 1, 128, 4, 64, 64, 4, 64, "f32"),
        # DiffMamba ~130M mixer: d_model 768, expand 2 -> 24 heads x 64, per-head B/C
        Workload("mixer130m_b32_L1024", 32, 1024, 24, 64, 128, 24, 256, "bf16"),
        # the same shape at batch 4 and 8 (profiler captures of the backward
        # and of the mixer block, a few GB on the device)
        Workload("mixer130m_b4_L1024", 4, 1024, 24, 64, 128, 24, 256, "bf16"),
        Workload("mixer130m_b8_L1024", 8, 1024, 24, 64, 128, 24, 256, "bf16"),
        # the same with B/C shared by all heads (ngroups 1)
        Workload("mixer130m_b32_L1024_g1", 32, 1024, 24, 64, 128, 1, 256, "bf16"),
        # LM1B packed-128, batch 512, B/C shared across heads
        Workload("packed128_b512_g1", 512, 128, 24, 64, 128, 1, 64, "bf16"),
        # long-context full-sequence mixer
        Workload("long_L65536", 1, 65536, 32, 64, 128, 32, 256, "bf16"),
        # the same layout at 16384 tokens (~0.7 GB on the device: small enough
        # for a full profiler capture of the segmented path's kernels)
        Workload("long_L16384", 1, 16384, 32, 64, 128, 32, 256, "bf16"),
        # block-diffusion step: prefix of 262144 tokens, active block of 64, 32 steps
        Workload("blockstep_prefix262144_blk64", 4, 262144, 32, 64, 128, 32, 256, "bf16",
                 block=64, steps=32),
        # the same step behind a 16384-token prefix (~1 GB on the device: small
        # enough for a full profiler capture of the block-step kernels)
        Workload("blockstep_prefix16384_blk64", 4, 16384, 32, 64, 128, 32, 256, "bf16",
                 block=64, steps=32),
    ]
}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some sizes changed (for small parity cases)."""
    return replace(w, **kw)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _dt(g, shape, device):
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return torch.nn.functional.softplus(z - 4.0).clamp_(1e-3, 0.1)


def _A(g, n, device):
    u = torch.rand(n, generator=g, device=device, dtype=torch.float32)
    u = u * (math.log(16.0) - math.log(1.0)) + math.log(1.0)
    return -torch.exp(u)


def _bc(g, shape, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) / 8.0


def bidir_inputs(batch, seqlen, nheads, headdim, dstate, ngroups, dtype="bf16",
                 seed=0, device="cpu"):
    """Inputs of one bidirectional mixer call, direction-stacked:
    x (batch,L,H,P); dt (2,batch,L,H); A (2,H) fp32; B, C (2,batch,L,G,N); D (2,H) fp32."""
    io = DTYPES[dtype]
    g = _gen(device, seed)
    x = torch.randn(batch, seqlen, nheads, headdim, generator=g, device=device)
    dts, As, Bs, Cs, Ds = [], [], [], [], []
    for _d in range(2):
        dts.append(_dt(g, (batch, seqlen, nheads), device))
        As.append(_A(g, nheads, device))
        Bs.append(_bc(g, (batch, seqlen, ngroups, dstate), device))
        Cs.append(_bc(g, (batch, seqlen, ngroups, dstate), device))
        Ds.append(torch.randn(nheads, generator=g, device=device))
    return dict(
        x=x.to(io), dt=torch.stack(dts).to(io), A=torch.stack(As).float().contiguous(),
        B=torch.stack(Bs).to(io), C=torch.stack(Cs).to(io),
        D=torch.stack(Ds).float().contiguous())


def workload_inputs(w: Workload, seed=0, device="cpu"):
    return bidir_inputs(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                        w.dtype, seed=seed, device=device)


def blockstep_inputs(batch, prefix_len, block, steps, nheads, headdim, dstate, ngroups,
                     dtype="bf16", seed=0, device="cpu"):
    """Inputs of a block-diffusion run.

    Draw order: per direction (A, D); then the prefix (x, forward dt, forward B);
    then, for every denoising step, a fresh block (x, dt[2], B[2], C[2]).
    Returns dict(A (2,H), D (2,H), x_pre (batch,Lp,H,P), dt_pre (batch,Lp,H),
    B_pre (batch,Lp,G,N), steps=[dict(x, dt, B, C) per step])."""
    io = DTYPES[dtype]
    g = _gen(device, seed)
    As, Ds = [], []
    for _d in range(2):
        As.append(_A(g, nheads, device))
        Ds.append(torch.randn(nheads, generator=g, device=device))
    x_pre = torch.randn(batch, prefix_len, nheads, headdim, generator=g, device=device).to(io)
    dt_pre = _dt(g, (batch, prefix_len, nheads), device).to(io)
    B_pre = _bc(g, (batch, prefix_len, ngroups, dstate), device).to(io)
    st = []
    for _k in range(steps):
        xb = torch.randn(batch, block, nheads, headdim, generator=g, device=device).to(io)
        dtb = torch.stack([_dt(g, (batch, block, nheads), device) for _ in range(2)]).to(io)
        Bb = torch.stack([_bc(g, (batch, block, ngroups, dstate), device) for _ in range(2)]).to(io)
        Cb = torch.stack([_bc(g, (batch, block, ngroups, dstate), device) for _ in range(2)]).to(io)
        st.append(dict(x=xb, dt=dtb, B=Bb, C=Cb))
    return dict(A=torch.stack(As).float().contiguous(), D=torch.stack(Ds).float().contiguous(),
                x_pre=x_pre, dt_pre=dt_pre, B_pre=B_pre, steps=st)


def to_f64(t):
    """Exact float64 copy of a (possibly bf16, possibly device) tensor as numpy."""
    return t.detach().to("cpu", torch.float64).numpy()


def block_inputs(w: Workload, conv_k: int = 4, seed=0, device="cpu"):
    """Inputs of the mixer block (ssd_mixer_block_fwd) at a workload's sizes.

    Draw order: xbc (the projected x, B, C channels) ~ N(0, 1), z ~ N(0, 1),
    dt_raw (2, batch, L, H) ~ N(0, 1); then per direction: conv_w (Cin, K)
    and conv_b (Cin) ~ U(-1/sqrt(K), 1/sqrt(K)) (the usual depthwise conv
    initialisation), dt_bias (H) ~ U(-7, -2.3), A = -exp(U(log 1, log 16)),
    D ~ N(0, 1); norm_w = 1. Activations are rounded to the I/O dtype;
    parameters are fp32."""
    io = DTYPES[w.dtype]
    g = _gen(device, seed)
    HP, GN = w.nheads * w.headdim, w.ngroups * w.dstate
    cin = HP + 2 * GN
    xbc = torch.randn(w.batch, w.seqlen, cin, generator=g, device=device).to(io)
    z = torch.randn(w.batch, w.seqlen, w.nheads, w.headdim, generator=g, device=device).to(io)
    dt_raw = torch.randn(2, w.batch, w.seqlen, w.nheads, generator=g, device=device).to(io)
    bound = 1.0 / (conv_k ** 0.5)
    cw, cb, db, As, Ds = [], [], [], [], []
    for _d in range(2):
        cw.append((torch.rand(cin, conv_k, generator=g, device=device) * 2 - 1) * bound)
        cb.append((torch.rand(cin, generator=g, device=device) * 2 - 1) * bound)
        db.append(torch.rand(w.nheads, generator=g, device=device) * 4.7 - 7.0)
        As.append(_A(g, w.nheads, device))
        Ds.append(torch.randn(w.nheads, generator=g, device=device))
    return dict(xbc=xbc, z=z, dt_raw=dt_raw, conv_w=torch.stack(cw).contiguous(), conv_b=torch.stack(cb).contiguous(),
                dt_bias=torch.stack(db).contiguous(), A=torch.stack(As).float().contiguous(),
                D=torch.stack(Ds).contiguous(), norm_w=torch.ones(HP, device=device))
