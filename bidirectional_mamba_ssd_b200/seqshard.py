"""The bidirectional mixer over sequences split across the ranks of a process
group (one GPU per rank).

Rank r holds tokens [r * Ls, (r + 1) * Ls) of every sequence, the same Ls on
every rank, and gets back the mixer's output for those tokens. Per call:

  1. ssd_segment_states: the local segment's forward state after its last
     token and reverse state before its first token, both from zero, and the
     two decays exp(A * sum of dt) over the segment (fused kernel);
  2. one all_gather over the group of those four (per (batch, head):
     2 x headdim x dstate + 2 fp32 values per rank);
  3. ssd_segment_carry for this rank's segment (the states the other
     segments leave), then ssd_bidir_fwd_seeded over the local tokens.

The recurrence is linear in the state, so the result is the mixer over the
whole sequence up to rounding (include/ssd_bidir.h, ssd_segment_states).
Every rank takes the same collective, once, in the same order. The exchange
is the only step between GPUs and it moves states, not tokens; the pages
describe no split across GPUs, only 65K- and 262K-token sequences ("Training
Hybrid Block Diffusion Language Models with Partial Bidirectionality", Key
Results).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import ssd_bidir_fwd_seeded, ssd_segment_carry, ssd_segment_states


class KernelOps:
    """The three per-rank steps, run by the library's kernels."""
    segment_states = staticmethod(ssd_segment_states)
    segment_carry = staticmethod(ssd_segment_carry)
    bidir_seeded = staticmethod(ssd_bidir_fwd_seeded)


def gather_segments(parts, group=None):
    """All-gather a list of tensors from every rank in one collective; returns
    one tensor per part with a leading rank dimension (segment-major)."""
    world = dist.get_world_size(group)
    flat = torch.cat([p.reshape(-1) for p in parts])
    bufs = [torch.empty_like(flat) for _ in range(world)]
    dist.all_gather(bufs, flat, group=group)
    out, off = [], 0
    for p in parts:
        n = p.numel()
        out.append(torch.stack([b[off:off + n].view(p.shape) for b in bufs]))
        off += n
    return out


def ssd_bidir_fwd_seq_sharded(x, dt, A, B, C, D, *, group=None, ops=None):
    """Mixer output for this rank's tokens of sequences split across `group`.

    x (batch, Ls, H, P), dt (2, batch, Ls, H), B/C (2, batch, Ls, G, N) are
    this rank's segment; A, D (2, H) are the same on every rank. Segment order
    is rank order."""
    ops = ops or KernelOps
    rank = dist.get_rank(group)
    fs, fd, rs, rd = ops.segment_states(x, dt, A, B)
    fs_all, fd_all, rs_all, rd_all = gather_segments([fs, fd, rs, rd], group)
    fwd_in, rev_in = ops.segment_carry(fs_all, fd_all, rs_all, rd_all, rank)
    return ops.bidir_seeded(x, dt, A, B, C, D, fwd_in, rev_in)
