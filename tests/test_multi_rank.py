"""Two-rank host logic of bench.py, on CPU with gloo.

With N GPUs the bench runs one process per GPU, each on its own replica of the
workload. Nothing crosses ranks on the data path. The ranks only meet at the
barrier that brackets the timed region, and at the all-reduce that takes the
slowest rank's time. These tests run that logic with two gloo ranks:
- the max over ranks;
- the whole-job rate;
- the reference arm returning at once on every rank but 0;
- the relaunch command used when --gpus N is given without torch.distributed.run;
- the agreement on a failed host-side leg: one rank's failure is seen by all ranks,
  which then all skip the leg's remaining collectives together.
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
        # a leg that failed on rank 1 only: both ranks learn it from the same all-reduce
        agreed = (bench.all_ranks_ok(dist, True), bench.all_ranks_ok(dist, r != 1))
        bench.barrier(dist)
    finally:
        dist.destroy_process_group()
    queue.put((rank, r, w, lr, slowest, rate, ref, agreed))


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
    for rank, (got_rank, r, w, lr, mx, rate, ref, agreed) in enumerate(results):
        assert (got_rank, r, w, lr) == (rank, rank, 2, rank)
        assert agreed == (True, False)
        assert mx == slowest
        assert rate == pytest.approx(2 * 100.0 / slowest)
    assert results[1][6] is None
    assert results[0][6] == "rank 0"


def test_single_rank_needs_no_process_group():
    assert bench.rank_env({}) == (0, 1, 0)
    assert bench.all_ranks_ok(None, True) and not bench.all_ranks_ok(None, False)
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


def test_device_failures_end_the_run():
    assert bench.is_device_failure(RuntimeError("CUDA error: an illegal memory access was encountered"))
    assert bench.is_device_failure(RuntimeError("device error during decode"))
    assert not bench.is_device_failure(MemoryError("pinned host buffer"))
    assert not bench.is_device_failure(ValueError("bad shape"))


def test_compact_summary_is_short_and_last_fields():
    pt = {"top_k": 16, "seq_len": 8192, "ms_per_step": 1.23456, "tflops": 654.321, "frac": 0.40111}
    line = {"ms_per_step": 4.56789, "value": 812.3456, "fwd_tflops": 1000.1, "bwd_tflops": 700.7,
            "frac_of_peak": {"step": 0.49812, "fwd": 0.6, "bwd": 0.43},
            "decode": {"tok_per_s": 612345.0, "ms_per_step": 0.0261234,
                       "roofline": {"achieved": 4567.8, "frac": 0.69861}},
            "sweep": {"points": [dict(pt, top_k=k, seq_len=n) for k in (16, 32, 64) for n in (8192, 32768, 65536)]
                      + [dict(pt, top_k=64, seq_len=131072)]},
            "long_decode": {"workloads": [{"batch": 1, "cache_len": 524288, "ms_per_step": 0.05, "select_share": 0.81}
                                          for _ in range(4)]}}
    out = bench.compact_summary(line)
    assert out["train"] == [4.57, 812.0, 0.498]
    assert out["decode"] == [612000.0, 26.1, 4570.0, 0.699]
    assert len(out["sweep"]) == 10 and out["sweep"][0] == [16, 8192, 1.23, 654.0, 0.401]
    import json
    assert len(json.dumps({"summary": out})) < 1200  # fits the tail a line reader keeps
