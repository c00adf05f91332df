"""The N>1 benchmark path (independent replicas, max-over-ranks timing) with
world_size 2 on CPU under gloo."""
import os
import socket

import torch.multiprocessing as mp

from semi_structured_sparse_02_b200 import replicas


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    replicas.init("gloo", rank, timeout_s=30)
    replicas.barrier()
    t = 1.0 + rank * 0.5  # rank 1 is the slow replica
    tmax = replicas.max_over_ranks(t)
    rate = replicas.aggregate_rate(100.0, tmax, world)
    out[rank] = (tmax, rate)
    replicas.barrier()
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == out[1] == (1.5, 2 * 100.0 / 1.5)


def test_single_process_needs_no_group():
    assert replicas.max_over_ranks(3.25) == 3.25
    assert replicas.aggregate_rate(10.0, 2.0, 1) == 5.0
