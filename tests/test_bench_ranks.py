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


def test_launch_plan_honours_gpus():
    import bench
    assert bench.launch_plan(1, {}) == ("run", 1)
    assert bench.launch_plan(2, {}) == ("spawn", None)
    assert bench.launch_plan(4, {"WORLD_SIZE": "4"}) == ("run", 4)
    assert bench.launch_plan(2, {"WORLD_SIZE": "1"})[0] == "error"
    assert bench.launch_plan(1, {"WORLD_SIZE": "8"})[0] == "error"
    assert bench.launch_plan(0, {})[0] == "error"


def _run_bench(args, env_extra=None, timeout=150):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env.update(env_extra or {})
    p = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], env=env,
                       capture_output=True, text=True, timeout=timeout, cwd=root)
    lines = [json.loads(x) for x in p.stdout.splitlines() if x.startswith("{")]
    return p.returncode, lines, p.stderr


@pytest.mark.timeout(200)
def test_gpus_two_without_launcher_starts_two_ranks():
    # bench.py --gpus 2 with no torchrun around it starts two local ranks
    # itself (gloo in the dry run) and rank 0 alone prints the line
    rc, lines, err = _run_bench(["--gpus", "2", "--dry-run", "--steps", "3", "--warmup", "3"])
    assert rc == 0, err
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and sorted(lines[0]["ranks"]) == [0, 1]
    assert lines[0]["max_over_ranks"] == 2.0


@pytest.mark.timeout(100)
def test_gpus_mismatch_with_launcher_fails_loudly():
    rc, lines, err = _run_bench(["--gpus", "2", "--dry-run"], {"WORLD_SIZE": "1"})
    assert rc != 0 and not lines
    assert "--gpus 2" in err
