"""Two-rank host logic of bench.py, on CPU with gloo.

With N GPUs the bench runs one process per GPU, each on its own replica of the
workload. Nothing crosses ranks on the data path. The ranks only meet at the
barrier that brackets the timed region, and at the all-reduce that takes the
slowest rank's time. These tests run that logic with two gloo ranks:
- the max over ranks;
- the whole-job rate;
- the reference arm returning at once on every rank but 0;
- the relaunch command used when --gpus N is given without torch.distributed.run.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _Args:
    steps, warmup = 1, 3


def _worker(rank: int, world: int, port: int, times, queue) -> None:
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    r, w, lr = bench.rank_env()
    dist = bench.init_ranks(w, "gloo", timeout_s=60)
    try:
        bench.barrier(dist)
        slowest = bench.max_over_ranks(dist, times[rank])
        rate = bench.job_rate(100.0, w, slowest)
        # every rank but 0 leaves the reference arm at once, without work
        ref = bench.run_reference(_Args(), r, w) if r != 0 else "rank 0"
        bench.barrier(dist)
    finally:
        dist.destroy_process_group()
    queue.put((rank, r, w, lr, slowest, rate, ref))


@pytest.mark.parametrize("times", [(3.0, 5.0), (7.5, 2.0)])
def test_two_ranks_take_the_slowest_time(times):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(rank, 2, port, times, queue)) for rank in range(2)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = max(times)
    for rank, (got_rank, r, w, lr, mx, rate, ref) in enumerate(results):
        assert (got_rank, r, w, lr) == (rank, rank, 2, rank)
        assert mx == slowest
        assert rate == pytest.approx(2 * 100.0 / slowest)
    assert results[1][6] is None
    assert results[0][6] == "rank 0"


def test_single_rank_needs_no_process_group():
    assert bench.rank_env({}) == (0, 1, 0)
    assert bench.init_ranks(1, "gloo") is None
    assert bench.max_over_ranks(None, 4.25) == 4.25
    assert bench.job_rate(10.0, 1, 2.0) == 5.0


def test_relaunch_command_runs_one_rank_per_gpu():
    cmd = bench.relaunch_command(4, ["--steps", "5"], 29511)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[cmd.index("--master-port") + 1] == "29511"
    assert cmd[-3].endswith("bench.py") and cmd[-2:] == ["--steps", "5"]
