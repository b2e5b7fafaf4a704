"""The benchmark's cross-rank reductions (max of per-rank times, sum of
per-rank work) on two gloo ranks on the CPU -- the same calls bench.py makes
over NCCL when it runs N replicas."""

import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    bench.dist_init(w, "gloo")
    try:
        ms = bench.reduce_scalar(10.0 + rank, "max", w, "cpu")
        work = bench.reduce_scalar(100.0 * (rank + 1), "sum", w, "cpu")
        bench.barrier(w)
        results[rank] = (ms, work)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_time_and_summed_work():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        for r in range(world):
            assert results[r] == (11.0, 300.0)


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_scalar(3.5, "max", 1, "cpu") == 3.5
    assert bench.reduce_scalar(3.5, "sum", 1, "cpu") == 3.5
