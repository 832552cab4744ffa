"""The bench's multi-rank path on the CPU: world_size-2 gloo process groups
stand in for the NCCL ranks of `bench.py --gpus N` (one replica per GPU, no
data-path collective; the job's time is the slowest rank's)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, local_ms, out):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()                                   # the bench's barrier before timing
        ms = bench.max_over_ranks(local_ms[rank], dist, torch.device("cpu"))
        value = bench.job_throughput(4096 * 4096, world, 5, ms)
        dist.barrier()                                   # and after
        out.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    local_ms = [31.5, 33.25]
    procs = [ctx.Process(target=_rank, args=(r, world, port, local_ms, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(out.get(timeout=5) for _ in range(world))
    assert [r[1] for r in res] == [33.25, 33.25]          # every rank sees the max
    want = 4096 * 4096 * 2 * 5 / (33.25 / 1e3)
    assert all(r[2] == pytest.approx(want, rel=1e-12) for r in res)


def test_single_process_time_is_its_own():
    assert bench.max_over_ranks(12.5, None, torch.device("cpu")) == 12.5
    assert bench.job_throughput(100, 1, 4, 2.0) == pytest.approx(100 * 4 / 2e-3)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    """Under torchrun the reference arm runs on rank 0 alone; the other
    ranks exit 0 without output."""
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"steps": 1, "warmup": 0, "gpus": 2})()
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
