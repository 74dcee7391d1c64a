"""The benchmark's N > 1 path on CPU: two gloo ranks, each with its own
independent batch, device time taken as the max over ranks and throughput
counted over the units all ranks processed (no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import ssd_inputs as si
        local_ms = [3.0, 5.0][rank]
        job_ms = bench.job_time_ms(local_ms, world, "cpu")
        value = bench.job_throughput(1000, 4, world, job_ms)
        w = si.scaled(si.WORKLOADS["mixer130m_b32_L1024"], batch=1, seqlen=16, nheads=2)
        x = si.workload_inputs(w, seed=bench.rank_seed(rank))["x"]
        q.put((rank, job_ms, value, float(x.float().sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_whole_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert res[0][1] == res[1][1] == 5.0                 # max over ranks
    assert res[0][2] == res[1][2] == 1000 * 2 * 4 / 5e-3  # all ranks' units / job time
    assert res[0][3] != res[1][3]                        # independent batches per rank
