"""The multi-GPU host logic of bench.py on CPU: two gloo ranks (no GPU).

Each rank scores its own problem (weak scaling), the step time is the max
over ranks, and the whole-job throughput counts every rank's units.
"""
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


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_init("gloo")
    assert (w, r) == (world, rank)
    local_ms = 10.0 + 5.0 * rank           # rank 1 is the slow one
    bench.barrier(w)
    ms = bench.max_over_ranks(local_ms, w)
    seed = bench.rank_seed(3, r)
    value = bench.job_throughput(1000, w, ms)
    out.put((r, ms, seed, value))
    dist.destroy_process_group()


def test_two_gloo_ranks_share_the_max_time_and_own_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, s0, v0), (r1, ms1, s1, v1) = res
    assert (r0, r1) == (0, 1)
    assert ms0 == ms1 == 15.0                      # max over ranks on every rank
    assert s0 != s1                                # independent problems per rank
    assert v0 == v1 == pytest.approx(2 * 1000 / 0.015)   # whole job: both ranks' units


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(10, 1, 1000.0) == 10.0
    assert bench.rank_seed(3, 0) == 1003
