"""The N > 1 path of bench.py on CPU: two gloo ranks.

The path shards by sequence (independent replicas, weak scaling): the only
collectives are the barrier and the max over ranks of the device timings, and
the whole-job value is the units of all ranks over the slowest rank's time.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, ws: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    sys.path.insert(0, ROOT)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from kv_cache_mtla_b200 import inputs

        bench._barrier(ws)
        # each rank's own step time; the job is as slow as the slowest rank
        local_ms = 10.0 + 5.0 * rank
        max_ms = bench._max_over_ranks(local_ms, ws)
        value = bench.job_value(1000.0, ws, 4, max_ms)
        # independent replicas: every rank draws its own sequences
        wl = bench.WL.with_(seed=bench.WL.seed + 1000 * rank)
        tok = inputs.tokens(wl, 8, stream=0)["c"]
        digest = float(tok.double().sum())
        q.put((rank, max_ms, value, digest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_as_weak_scaling():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(q.get(timeout=5) for _ in range(ws))
    # every rank sees the same max, and the job value divides all ranks' units by it
    assert [g[1] for g in got] == [15.0, 15.0]
    expect = 1000.0 * ws * 4 / (15.0 / 1e3)
    assert all(g[2] == pytest.approx(expect) for g in got)
    # the two replicas are different sequences
    assert got[0][3] != got[1][3]


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench._max_over_ranks(3.5, 1) == 3.5
    assert bench.job_value(100.0, 1, 2, 1000.0) == pytest.approx(200.0)
    assert torch.isfinite(torch.tensor(bench.job_value(1.0, 8, 1, 0.5)))
