"""The sequence-sharded mixer's exchange on CPU: gloo ranks each holding one
segment of every sequence run seqshard.ssd_bidir_fwd_seq_sharded with the
per-rank steps done by the fp64 oracle (test infrastructure) instead of the
GPU kernels. What is under test is the host side: the single all_gather of
the segment states, its segment-major unpacking, the rank-to-segment order
and the carried states. Each rank checks the states carried into its segment
against the oracle's states of the whole prefix and suffix, and its output
against the oracle's mixer over the whole sequence."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

SEG = 7


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _problem(world):
    rng = np.random.default_rng(31)
    batch, L, H, P, N, G = 2, SEG * world, 4, 3, 5, 2
    x = rng.standard_normal((batch, L, H, P))
    dt = rng.uniform(0.05, 0.6, size=(2, batch, L, H))
    A = -rng.uniform(0.2, 2.0, size=(2, H))
    B = rng.standard_normal((2, batch, L, G, N))
    C = rng.standard_normal((2, batch, L, G, N))
    D = rng.standard_normal((2, H))
    return x, dt, A, B, C, D


def _flip(a):
    return np.flip(a, axis=1).copy()


class OracleOps:
    """The per-rank steps on the CPU, from their definitions (fp64)."""

    @staticmethod
    def segment_states(x, dt, A, B):
        import oracle
        x, dt, A, B = (t.numpy() for t in (x, dt, A, B))
        fs = oracle.prefix_state(x, dt[0], A[0], B[0])
        # the reverse scan over the segment is a forward scan of the flipped segment
        rs = oracle.prefix_state(_flip(x), _flip(dt[1]), A[1], _flip(B[1]))
        fd = np.exp(A[0][None, :] * dt[0].sum(axis=1))
        rd = np.exp(A[1][None, :] * dt[1].sum(axis=1))
        return tuple(torch.from_numpy(np.ascontiguousarray(a)) for a in (fs, fd, rs, rd))

    @staticmethod
    def segment_carry(fs, fd, rs, rd, seg):
        nseg = fs.shape[0]
        f = torch.zeros_like(fs[0])
        for q in range(seg):
            f = fd[q][..., None, None] * f + fs[q]
        r = torch.zeros_like(rs[0])
        for q in range(nseg - 1, seg, -1):
            r = rd[q][..., None, None] * r + rs[q]
        return f, r

    @staticmethod
    def bidir_seeded(x, dt, A, B, C, D, fwd_in, rev_in):
        import oracle
        y = oracle.bidir_seeded(*(t.numpy() for t in (x, dt, A, B, C, D)), fwd_in.numpy(), rev_in.numpy())
        return torch.from_numpy(y)


class CheckedOps(OracleOps):
    """OracleOps that also hands the carried states back for checking."""
    seen = {}

    @classmethod
    def segment_carry(cls, fs, fd, rs, rd, seg):
        f, r = OracleOps.segment_carry(fs, fd, rs, rd, seg)
        cls.seen["carry"] = (f.numpy().copy(), r.numpy().copy())
        return f, r


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from bidirectional_mamba_ssd_b200 import seqshard
        x, dt, A, B, C, D = _problem(world)
        t0, t1 = rank * SEG, (rank + 1) * SEG
        local = [torch.from_numpy(np.ascontiguousarray(a)) for a in
                 (x[:, t0:t1], dt[:, :, t0:t1], A, B[:, :, t0:t1], C[:, :, t0:t1], D)]
        y = seqshard.ssd_bidir_fwd_seq_sharded(*local, ops=CheckedOps).numpy()
        full = oracle.bidir(x, dt, A, B, C, D)[:, t0:t1]
        f_in, r_in = CheckedOps.seen["carry"]
        # the states the rest of the sequence leaves, straight from the oracle
        f_ref = oracle.prefix_state(x[:, :t0], dt[0][:, :t0], A[0], B[0][:, :t0]) if t0 > 0 else np.zeros_like(f_in)
        if t1 < x.shape[1]:
            r_ref = oracle.prefix_state(_flip(x[:, t1:]), _flip(dt[1][:, t1:]), A[1], _flip(B[1][:, t1:]))
        else:
            r_ref = np.zeros_like(r_in)
        rel = lambda a, b: float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))
        q.put((rank, rel(y, full), float(np.max(np.abs(f_in - f_ref))), float(np.max(np.abs(r_in - r_ref)))))
    finally:
        dist.destroy_process_group()


def _run(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_two_ranks_rebuild_the_whole_sequence():
    for rank, err, ferr, rerr in _run(2):
        assert err < 1e-12, (rank, err)
        assert ferr < 1e-12 and rerr < 1e-12, (rank, ferr, rerr)


def test_three_ranks_middle_segment_takes_states_from_both_sides():
    res = _run(3)
    assert [r[0] for r in res] == [0, 1, 2]
    for rank, err, ferr, rerr in res:
        assert err < 1e-12, (rank, err)
        assert ferr < 1e-12 and rerr < 1e-12, (rank, ferr, rerr)
