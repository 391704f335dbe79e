"""The multi-GPU bookkeeping of bench.py on CPU: two gloo ranks, each with its
own independent problem, must agree on the max-over-ranks time and the
whole-job (weak-scaling) throughput.  No GPU and no collective on the data
path: the only exchange is the timing reduction."""
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


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    try:
        ws, r, _ = bench.dist_env()
        assert (ws, r) == (world, rank)
        # rank-dependent per-step times: the slowest rank decides
        ms, launch = bench.max_over_ranks([1.0 + rank, 0.5 + 0.25 * rank], torch.device("cpu"))
        value = bench.aggregate_throughput(52.3e9, ms, ws)
        out_q.put((rank, ms, launch, value))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_and_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, launch, value in res:
        assert ms == 2.0 and launch == 0.75
        assert value == pytest.approx(world * 52.3e9 / 2.0e-3 / 1e12)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.0], torch.device("cpu")) == [3.0, 4.0]
    assert bench.aggregate_throughput(1e12, 1000.0, 1) == pytest.approx(1.0)
