"""The bench's several-GPU path on CPU ranks (gloo, world size 2): the path has no
data-path exchange (replicas only), so the ranks only meet to combine their
timings: the slowest rank's time and the sum of all ranks' work."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        ms = [12.5, 20.0][rank]         # rank 1 is slower
        work = [3.0, 5.0][rank]
        out = bench.reduce_over_ranks(dist, torch.device("cpu"), ms, work, ms * 2, work / 2)
        dist.barrier()
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_two_cpu_ranks_combine_timings_as_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        ms_max, work_sum, ms_e_max, work_e_sum = res[r]
        assert ms_max == 20.0 and work_sum == 8.0 and ms_e_max == 40.0 and work_e_sum == 4.0


def test_single_rank_keeps_its_own_figures():
    import bench
    assert bench.reduce_over_ranks(None, None, 1.0, 2.0, 3.0, 4.0) == (1.0, 2.0, 3.0, 4.0)
