"""The multi-rank path of bench.py (replicas, one per GPU) on CPU with the gloo backend: every rank
reports its own device time, all ranks agree on the max, and the whole-job value counts every rank's
points.  Two ranks, 127.0.0.1 rendezvous, a short process-group timeout."""
import datetime
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


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    import bench
    local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
    dist.barrier()
    total = bench.reduce_max(local_ms, dist, "cpu")
    value = bench.aggregate_value(world, 2, 65536, 100, total)
    out.put((rank, total, value))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]           # both ranks see the slowest rank's time
    want = 2 * 2 * 65536 * 100 / 15e-3                   # every rank's points, over the max time
    assert all(abs(r[2] - want) < 1e-6 * want for r in res)


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max(3.5) == 3.5
    assert bench.aggregate_value(1, 2, 10, 5, 1000.0) == 100.0


def _rank_dies(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    import bench
    dist.barrier()  # the warm-up steps end together
    if rank == 1:
        os._exit(3)  # this rank leaves between steps, with nothing of its own in flight
    try:
        bench.reduce_max(10.0, dist, "cpu")  # the timed region's max over ranks
        out.put((rank, "returned"))
    except Exception as e:  # the peer is gone: the collective ends with an error instead of waiting for ever
        out.put((rank, "error: " + type(e).__name__))
    out.close()
    out.join_thread()  # the result is on its way to the parent before this process leaves
    os._exit(0)


def test_a_rank_that_leaves_is_an_error_not_a_hang():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_dies, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    rank, what = out.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert rank == 0 and what.startswith("error"), what
    assert procs[1].exitcode == 3
