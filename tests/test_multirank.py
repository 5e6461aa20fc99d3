"""The multi-GPU host logic of bench.py, run as two gloo ranks on the CPU.

With N GPUs every rank runs its own batch of the workload (weak scaling,
no collective on the data path); the ranks only agree on the timed region
(the slowest rank's time) and rank 0 reports the whole job's throughput.
These tests run that agreement with world size 2 over gloo.
"""
import datetime
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # each rank's own step time; the timed region is the slowest rank's
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
        out.put((rank, ms, bench.rank_seed(2, rank, world)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time_and_use_distinct_batches():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=5) for _ in range(2))
    assert [r[1] for r in res] == [15.0, 15.0]
    seeds = [r[2] for r in res]
    assert seeds[0] != seeds[1]


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, 1, torch.device("cpu")) == 3.25
    assert bench.rank_seed(2, 0, 1) == 2 and bench.rank_seed(5, 0, 1) == 5


@pytest.mark.parametrize("world", [1, 2, 8])
def test_whole_job_value_is_weak_scaling_sum(world):
    # every rank did 1.5e12 FLOPs in (at most) 1.5 ms: 1000 TFLOP/s per rank
    assert bench.whole_job_value(1.5e12, world, 1.5) == pytest.approx(1000.0 * world)


def test_gpus_flag_must_match_the_launched_world_size():
    """Under torchrun the rank count comes from WORLD_SIZE; a --gpus that
    disagrees is an error (exit 2) before any GPU work, not a silent 1-GPU run."""
    import subprocess
    import sys
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, bench.__file__, "--gpus", "2", "--steps", "1"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 2, (r.returncode, r.stderr[-500:])
    assert "WORLD_SIZE is 1" in r.stderr


def test_gpus_flag_without_torchrun_starts_that_many_ranks(monkeypatch):
    """--gpus N > 1 outside torchrun re-runs the script under
    torch.distributed.run with N processes on 127.0.0.1."""
    import subprocess
    seen = {}
    monkeypatch.setattr(subprocess, "call", lambda cmd: seen.setdefault("cmd", cmd) and 0)
    assert bench.relaunch_with_ranks(4) == 0
    cmd = seen["cmd"]
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
