"""The multi-rank host logic of bench.py on CPU: two gloo ranks time different totals,
the job's time is the slowest rank's, the whole-job throughput counts every rank's batch,
and the reference arm prints from rank 0 only."""
import datetime
import io
import os
import socket
import sys
import types
from contextlib import redirect_stdout

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # rank r "timed" 10 + r ms for its steps and 30 - r ms end to end
        tot, e2e = bench.reduce_max_over_ranks([10.0 + rank, 30.0 - rank], torch.device("cpu"))
        value = bench.job_throughput(1000, 4, world, tot)
        q.put((rank, tot, e2e, value))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_count_every_batch():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, tot, e2e, value in got:
        assert tot == 11.0                     # max over ranks of 10 + r
        assert e2e == 30.0                     # max over ranks of 30 - r
        assert value == pytest.approx(1000 * 4 * world / 0.011)


def test_reference_arm_prints_from_rank_zero_only():
    sys.path.insert(0, ROOT)
    import bench
    args = types.SimpleNamespace(gpus=2, steps=1, warmup=1)
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(args, rank=1) == 0
    assert buf.getvalue() == ""
