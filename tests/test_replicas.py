"""The multi-process path of bench.py on CPU: world size 2 over gloo.

`bench.py --gpus N` runs N independent replicas (the path has no exchange
step); what crosses ranks is only a barrier around the timed region and the
max over ranks of the elapsed time, from which rank 0 reports the whole-job
throughput.  These tests run that host logic with two gloo ranks."""
from __future__ import annotations

import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, q):
    import datetime
    import time

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(ws)
        t0 = time.perf_counter()
        time.sleep(0.05 * (rank + 1))  # rank 1 is the slow replica
        ms = (time.perf_counter() - t0) * 1e3
        bench.barrier(ws)
        ms_max = bench.allreduce_max(ws, ms, device="cpu")
        q.put((rank, ms, ms_max, bench.replica_throughput(1000, ms_max, 1, ws)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas_take_the_slowest_rank():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(2))
    (r0, ms0, max0, v0), (r1, ms1, max1, v1) = res
    assert (r0, r1) == (0, 1)
    assert ms1 > ms0
    assert max0 == max1 == pytest.approx(max(ms0, ms1))
    # whole-job value: both ranks' units over the slowest rank's time, identical on every rank
    assert v0 == v1 == pytest.approx(2 * 1000 / (max1 * 1e-3))


def test_single_process_helpers_are_identities():
    import bench
    assert bench.allreduce_max(1, 3.5, device="cpu") == 3.5
    bench.barrier(1)
    assert bench.replica_throughput(10, 1000.0, 2, 1) == pytest.approx(20.0)
