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


def _shard_rank(rank, world, port, out, seq_lens=(300, 1, 257), group=8):
    """One rank of a query-sharded indexer job, with the CPU oracle standing
    in for the per-rank compute: its range of query rows, then the gather."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import torch.distributed as dist

    import bench
    import oracle
    from long_context_sparse_misa_b200 import sharding
    from misa_synth import make_workload
    bench.dist_init("gloo")
    wl = make_workload(seq_lens=list(seq_lens), queries="all", H=8, B=16, m=4, k=20, seed=77)
    ranges = sharding.query_ranges(wl.q_pos, world, group=group)
    lo, hi = ranges[rank]
    # the shard's problem description is the workload's row subset
    sl, qo, qp = sharding.shard_metadata(wl.seq_lens, wl.query_offsets, wl.q_pos, lo, hi)
    sub = wl.subset_queries(range(lo, hi))
    assert np.array_equal(qo, sub.query_offsets) and np.array_equal(qp, sub.q_pos)
    assert np.array_equal(sl, wl.seq_lens)
    rows = oracle.misa_index(sub)["rows"]
    idx = torch.from_numpy(np.stack([r["idx"] for r in rows])) if rows else \
        torch.zeros((0, wl.k), dtype=torch.int32)
    val = torch.from_numpy(np.stack([r["val"] for r in rows])) if rows else \
        torch.zeros((0, wl.k), dtype=torch.float64)
    g_idx = sharding.gather_rows(idx, ranges)
    g_val = sharding.gather_rows(val, ranges)
    full = oracle.misa_index(wl)["rows"]
    ok = (np.array_equal(g_idx.numpy(), np.stack([r["idx"] for r in full])) and
          np.array_equal(g_val.numpy(), np.stack([r["val"] for r in full])))
    out.put((rank, hi - lo, ok))
    dist.destroy_process_group()


def test_query_sharded_oracle_gathers_to_the_unsharded_result():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok for _, _, ok in res)
    assert sum(n for _, n, _ in res) == 558 and all(n > 0 for _, n, _ in res)


def test_query_sharded_oracle_with_an_empty_rank():
    # 27 queries over three ranks in 8-row groups: ranges [0,16) [16,16) [16,27),
    # so rank 1 holds no query and rank 2 spans a sequence boundary; the padded
    # all_gather still gives every rank the unsharded result.
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_rank, args=(r, 3, port, q, (24, 3), 8)) for r in range(3)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok for _, _, ok in res)
    assert [n for _, n, _ in res] == [16, 0, 11]


def test_query_ranges_balance_causal_work():
    import numpy as np
    sys.path.insert(0, ROOT)
    from long_context_sparse_misa_b200 import sharding
    q_pos = np.arange(131072, dtype=np.int32)          # one 128K prefill
    for world in (1, 2, 4, 8):
        ranges = sharding.query_ranges(q_pos, world)
        assert ranges[0][0] == 0 and ranges[-1][1] == len(q_pos)
        assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
        assert all(lo % 32 == 0 for lo, _ in ranges)
        work = [int(np.sum(q_pos[lo:hi].astype(np.int64) + 1)) for lo, hi in ranges]
        assert max(work) / min(work) < 1.01
    # fewer rows than ranks: empty ranges, still a cover
    ranges = sharding.query_ranges(np.arange(5), 4, group=8)
    assert ranges[0][0] == 0 and ranges[-1][1] == 5
    assert sum(hi - lo for lo, hi in ranges) == 5
