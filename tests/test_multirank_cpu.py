"""Host logic of the multi-GPU bench path on CPU: two gloo ranks, max and sum over ranks
(the bench times every rank and reports the slowest, with the work of all ranks)."""
import os
import socket

import pytest
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
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    mx = bench.max_over_ranks(10.0 + rank * 3.5, world, "cpu")
    sm = bench.sum_over_ranks(4096.0, world, "cpu")
    q.put((rank, mx, sm))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_and_sum_over_two_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(100)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, mx, sm in got:
        assert mx == 13.5 and sm == 8192.0


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0 and bench.sum_over_ranks(2.0, 1) == 2.0
