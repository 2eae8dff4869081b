"""The multi-GPU bench path runs one independent replica per rank (the layer does not shard).
Its host logic is checked here on CPU with two gloo ranks: every rank sees the slowest rank's
time, the rate counts the tokens of all ranks, and only rank 0 reports."""
import contextlib
import datetime
import io
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, rank_ms, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(rank_ms[rank], world, "cpu")
        q.put((rank, ms, bench.job_rate(1, 100, world, ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank_and_all_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    rank_ms = [3.0, 5.0]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, rank_ms, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, rate in got:
        assert ms == 5.0                       # max over ranks, on every rank
        assert abs(rate - 2 * 100 / 5e-3) < 1e-6   # both ranks' tokens over the slowest time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.job_rate(8, 10, 1, 2.0) == 8 * 10 / 2e-3


def test_reference_arm_prints_only_on_rank_zero():
    sys.path.insert(0, ROOT)
    import bench

    class A:
        workload, steps, warmup = "t1_int4_g64", 1, 0

    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(A(), rank=1, world=2)
    assert buf.getvalue() == ""
