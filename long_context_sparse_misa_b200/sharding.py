"""Query-axis sharding of one indexer problem over the ranks of a job.

Every query of the DSA / MISA indexer scores its own causal prefix and
selects its own top-k, so the queries of one long prefill are independent
given the keys ("MISA: Mixture of Indexer Sparse Attention for Long-Context
LLM Inference", gist.science summary, "Methodologie: MISA": routing and
token scoring are per query).  A job of R ranks therefore splits the query
rows into R contiguous ranges, each rank holds the whole key cache (K and
its pooled blocks are replicated), runs the indexer on its own range, and
the per-query results are gathered.  There is no other exchange.

The ranges balance causal work: query t costs about t + 1 scored pairs, so
the boundaries sit where the running sum of (q_pos + 1) crosses r / R of the
total, rounded to a multiple of `group` rows (the scorer's query groups of
the same sequence stay whole).  The contiguous ranges keep each rank's q and
w rows a plain slice of the caller's tensors.

Host logic only (plain numpy and torch.distributed); the per-rank compute is
the CUDA indexer of this package.
"""
from __future__ import annotations

import numpy as np

__all__ = ["query_ranges", "shard_metadata", "gather_rows"]


def query_ranges(q_pos, world: int, group: int = 32) -> list[tuple[int, int]]:
    """Contiguous query-row ranges [lo, hi), one per rank, with about equal
    sums of (q_pos + 1).  Boundaries are multiples of `group` rows (the last
    range ends at T).  Ranges may be empty when T is small."""
    q_pos = np.asarray(q_pos, dtype=np.int64)
    T = len(q_pos)
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = np.cumsum(q_pos + 1, dtype=np.float64)
    total = float(cost[-1]) if T else 0.0
    bounds = [0]
    for r in range(1, world):
        target = total * r / world
        cut = int(np.searchsorted(cost, target, side="left")) + 1 if T else 0
        cut = int(round(cut / group)) * group
        bounds.append(min(max(cut, bounds[-1]), T))
    bounds.append(T)
    return [(bounds[r], bounds[r + 1]) for r in range(world)]


def shard_metadata(seq_lens, query_offsets, q_pos, lo: int, hi: int):
    """Problem metadata of query rows [lo, hi): every sequence's keys (the
    key cache is replicated), the query offsets of the range and its
    positions.  Returns (seq_lens, query_offsets, q_pos) as numpy arrays."""
    qo = np.asarray(query_offsets, dtype=np.int64)
    shard_qo = (np.clip(qo, lo, hi) - lo).astype(np.int32)
    return (np.asarray(seq_lens, dtype=np.int64), shard_qo,
            np.asarray(q_pos, dtype=np.int32)[lo:hi].copy())


def gather_rows(local, ranges, group=None):
    """All ranks' result rows in query order, on every rank.

    local: this rank's rows, a torch tensor [hi - lo, ...] (its range of
    `ranges`); the ranges must cover 0..T contiguously in rank order.  Each
    rank pads its rows to the longest range, one all_gather moves them
    (NCCL over NVLink for CUDA tensors, gloo for CPU tensors), and the
    padding is dropped.  Returns a tensor [T, ...]."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if len(ranges) != world:
        raise ValueError("one range per rank")
    rows = max(hi - lo for lo, hi in ranges)
    pad = torch.zeros((rows,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:hi - lo] for p, (lo, hi) in zip(parts, ranges)], dim=0)
