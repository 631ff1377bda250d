"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

bench.py runs one replica per GPU (the DCA path has no exchange step); the only
cross-rank operations are a barrier around the timed region and the max over
ranks of the measured times, which decides the whole-job throughput.  These
run here with the gloo backend, no GPU involved.
"""

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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        bench._barrier(world)
        got = bench._max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        out[rank] = got
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_barrier_with_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_single_rank_needs_no_process_group():
    import bench
    assert bench._max_over_ranks(3.25, 1, torch.device("cpu")) == 3.25
    bench._barrier(1)
