"""The multi-rank host logic of bench.py on the CPU: two gloo processes.

bench.py --gpus N runs one process per GPU with no data-path collective (sequences are
independent): each rank decodes its own batch (seed + rank), the ranks meet at barriers and
the reported time is the maximum over ranks.  These tests run that plumbing with the gloo
backend on 127.0.0.1 and check the reference arm's rank-0-only rule.
"""

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    from paged_mla_decode_11_b200 import workloads as W
    g = bench.RankGroup("gloo", torch.device("cpu"))
    try:
        g.barrier()
        slowest = g.max(1.0 + rank)             # each rank's own step time
        x = W.make_inputs(W.TINY, seed=rank)   # each rank decodes its own batch
        g.barrier()
        results.put((rank, g.rank, g.world, slowest, float(x["q"].float().sum())))
    finally:
        g.close()


def test_two_gloo_ranks_barrier_and_max():
    world, port = 2, free_port()
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(results.get(timeout=5) for _ in range(world))
    assert [g[1] for g in got] == [0, 1] and all(g[2] == world for g in got)
    assert all(g[3] == 2.0 for g in got)            # maximum over ranks, seen by every rank
    assert got[0][4] != got[1][4]                   # different inputs per rank


def test_aggregate_is_whole_job():
    import bench
    # 2 ranks x 100 MB per step in 10 ms = 20 GB/s for the job
    assert bench.aggregate_throughput(100e6, 2, 0.01) == pytest.approx(20e9)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        workload, steps, warmup = "tiny", 1, 0

    assert bench.run_reference(Args()) is None
    assert capsys.readouterr().out == ""
