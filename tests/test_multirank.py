"""The multi-rank (replica) logic of bench.py on CPU: two gloo ranks.

The attention path shards into independent (batch, head) problems, so more
GPUs run replicas with no data exchange; the only collective is the max of
the device-timed step over ranks, which is what these ranks exercise."""

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


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + rank, 5.0 - rank]           # rank 1 is slower on the first value
        combined = bench.max_over_ranks(local)
        ws, r, _ = bench.dist_env()
        q.put((rank, combined, ws, r, bench.job_throughput(6.594e12, ws, combined[0])))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, combined, ws, r, tops in res:
        assert combined == [11.0, 5.0]               # element-wise max over ranks
        assert ws == 2 and r == rank
        assert tops == pytest.approx(2 * 6.594e12 / 11e-3 / 1e12)


def test_single_rank_is_identity():
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.job_throughput(1e12, 1, 1.0) == pytest.approx(1000.0)
