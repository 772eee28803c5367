"""The multi-process host logic of bench.py on CPU: two gloo ranks.

With N GPUs each rank runs an independent replica of the block; the bench
reports the slowest rank's time and sums the work of all ranks. These tests
run that aggregation over a real two-rank gloo process group, and check that
the reference arm prints only on rank 0.
"""

import contextlib
import io
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local = [100.0 + 10 * rank, 5.0 - rank]        # per-rank step time, attention time (ms)
        mx = bench.reduce_max(local, world)
        value = bench.job_throughput(7.0e13, 20, mx[0], world)
        out_q.put((rank, mx, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_aggregation():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, mx, value = q.get(timeout=120)
        results[rank] = (mx, value)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the maximum over ranks
    for rank in range(world):
        mx, value = results[rank]
        assert mx == [110.0, 5.0]
        # two replicas of 7e13 FLOP x 20 steps in 110 ms
        assert value == pytest.approx(2 * 7.0e13 * 20 / 0.110 / 1e12)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max([3.0, 1.0], 1) == [3.0, 1.0]
    assert bench.job_throughput(1e12, 10, 1000.0, 1) == pytest.approx(10.0)


def test_reference_arm_prints_only_on_rank_zero():
    sys.path.insert(0, ROOT)
    import bench
    from ulysses_sequence_attention_sp_b200.workloads import TINY

    class Args:
        steps, warmup, gpus = 1, 0, 2

    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(Args, TINY, rank=1, world=2)
    assert buf.getvalue() == ""
