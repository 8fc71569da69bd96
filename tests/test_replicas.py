"""Multi-process host logic of bench.py's replica mode (world size 2, gloo, CPU).

The decode step does not shard: `bench.py --gpus N` runs N independent replicas,
times each on its own device, and reports the slowest rank's time and the
whole-job throughput.  These tests run that host logic as two CPU processes.
"""
import os
import socket

import pytest

import bench


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, ws, port, out_q):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(ws)
        # rank r "took" 10 + 5 r ms for 4 steps
        mx = bench.max_over_ranks(ws, 10.0 + 5.0 * rank, device="cpu")
        bench.barrier(ws)
        out_q.put((rank, mx, bench.job_throughput(ws, 4, mx)))
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank_and_the_whole_job():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got.sort()
    assert [g[1] for g in got] == [15.0, 15.0]          # max over ranks, same on both
    assert got[0][2] == pytest.approx(2 * 4 / 0.015)    # 8 tokens in 15 ms


def test_single_rank_helpers_need_no_process_group():
    assert bench.max_over_ranks(1, 3.5) == 3.5
    bench.barrier(1)
    assert bench.job_throughput(1, 10, 20.0) == pytest.approx(500.0)
