"""The benchmark's multi-process path on CPU (gloo, world size 2).

The decode step shards by sequence with no exchange step, so `bench.py --gpus N` runs N
independent replicas; what the ranks share is the timing protocol: every rank's device
time is reduced with MAX and the value counts the units of all ranks.  These tests run
that protocol with two gloo ranks and check the reference arm's rank handling.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        args = bench.parse_args(["--gpus", str(world)])
        w, r, local = bench.dist_setup(args)
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, w)      # rank 1 is the slow one
        dist.barrier()
        q.put((r, w, local, slowest, bench.throughput(w, 1e9, 4, slowest)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 and r[2] == r[0] for r in res)
    assert all(r[3] == 15.0 for r in res)                 # max over ranks, seen by both
    # whole-job value: both replicas' bytes over the slowest rank's time
    assert all(abs(r[4] - 2 * 1e9 * 4 / 15e-3 / 1e9) < 1e-6 for r in res)


def test_single_process_reduction_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.throughput(1, 2e9, 10, 4.0) == pytest.approx(2e9 * 10 / 4e-3 / 1e9)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    args = bench.parse_args(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert bench.run_reference(args) == 0                 # returns at once, prints nothing
