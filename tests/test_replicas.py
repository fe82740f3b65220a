"""The multi-GPU path of the benchmark is N independent replicas (the layer
has no exchange step): only the barrier and the max-over-ranks timing cross
ranks.  Exercised here with world_size 2 on the gloo backend, on the CPU."""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    slowest = bench.max_over_ranks(1.5 + rank, device="cpu")
    v = bench.job_throughput(4096, 10, world, slowest)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, slowest, v))


def test_max_over_ranks_and_throughput_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, v in res:
        assert slowest == 2.5                      # the slower rank's time
        assert v == pytest.approx(2 * 4096 * 10 / 2.5)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, device="cpu") == 3.25
    assert bench.job_throughput(4096, 5, 1, 2.0) == 4096 * 5 / 2.0
