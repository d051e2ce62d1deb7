"""bench.py's multi-rank host logic on CPU: two gloo ranks stand in for two GPUs.

The path has no exchange step, so N GPUs run N independent replicas; what the
ranks share is the timing: every time is the slowest rank's, and the value is
the work of all ranks over that time.  The reference arm prints only on rank 0."""

import contextlib
import io
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # rank r measured (10 + r) ms for 4 steps, 2.0 + r ms per decode, 3.0 - r ms e2e
        ms_step, dec, e2e = bench._rank_times(10.0 + rank, 2.0 + rank, 3.0 - rank, 4, world)
        bench._barrier(world)
        value = bench._job_value(1000, world, ms_step)
        q.put((rank, ms_step, dec, e2e, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms_step, dec, e2e, value in res:
        assert ms_step == pytest.approx(11.0 / 4)      # max over ranks, per step
        assert dec == pytest.approx(3.0)
        assert e2e == pytest.approx(3.0)
        assert value == pytest.approx(1000 * 2 / (11.0 / 4 * 1e-3))


def test_single_rank_needs_no_process_group():
    import bench
    assert bench._rank_times(8.0, 1.0, 2.0, 4, 1) == (2.0, 1.0, 2.0)
    assert bench._job_value(500, 1, 2.0) == pytest.approx(250000.0)


def test_reference_arm_prints_only_on_rank_zero(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    args = bench.argparse.Namespace(workload="tiny", seed=0, warmup=0, steps=1, gpus=2)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args)
    assert buf.getvalue() == ""
