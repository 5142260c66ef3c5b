"""The decode step (B200 only): incremental pooling of the newest keys, and
the whole routed indexer step captured and replayed as one CUDA graph.

Incremental pooling re-pools only the blocks that hold new keys, with the
same arithmetic as the full pass, so the updated rows must be bit-identical
to a full re-pooling and every other row untouched.  A captured step must
give exactly what the same calls give when launched one by one.
"""
import numpy as np
import pytest
import torch

import long_context_sparse_misa_b200 as misa
from misa_synth import make_config, make_workload

pytestmark = pytest.mark.gpu


def _inputs(wl):
    prob = misa.Problem.from_workload(wl)
    return (prob, torch.from_numpy(wl.K_bits).cuda(), torch.from_numpy(wl.q_bits).cuda(),
            torch.from_numpy(wl.w).cuda())


def _status_ok():
    code, bits = misa.stream_status()
    assert code == 0 and bits == 0, f"device status {code}/{bits}"


def test_pool_from_matches_full_pooling_on_new_blocks_only():
    lens = [1000, 1537, 64, 129]
    wl = make_workload(seq_lens=lens, queries=1, H=8, B=64, m=8, k=16, seed=5)
    prob, K, _, _ = _inputs(wl)
    full = torch.empty((prob.total_blocks, 128), dtype=torch.float32, device="cuda")
    misa.pool_keys(prob, K, full)
    # new keys from these positions on; >= length means nothing new
    from_pos = [990, 1, 64, 129]
    bo = np.concatenate([[0], np.cumsum([(L + 63) // 64 for L in lens])])
    part = full.clone()
    stale = torch.zeros(prob.total_blocks, dtype=torch.bool)
    for s, (L, f) in enumerate(zip(lens, from_pos)):
        if f < L:
            stale[bo[s] + f // 64: bo[s + 1]] = True
    part[stale.cuda()] = float("nan")        # rows that must be recomputed
    kept = part[~stale.cuda()].clone()
    misa.pool_keys_from(prob, K, part, torch.tensor(from_pos, dtype=torch.int32, device="cuda"))
    _status_ok()
    assert torch.equal(part, full)                            # bit-identical
    assert torch.equal(part[~stale.cuda()], kept)             # others untouched


@pytest.mark.parametrize("cfg", [1, 4])
def test_decode_step_in_cuda_graph_equals_eager(cfg):
    wl = make_config(cfg)
    prob, K, q, w = _inputs(wl)
    ix = misa.Indexer(prob, m=wl.m, k=wl.k, k_cand=wl.k_cand)
    q_per_seq = np.diff(wl.query_offsets)
    new_from = torch.tensor(wl.seq_lens - q_per_seq, dtype=torch.int32, device="cuda")
    step = ((lambda: ix.hier(q, w, K, pool_from=new_from)) if wl.k_cand
            else (lambda: ix.misa(q, w, K, pool_from=new_from)))
    # eager: a full pooling first (the previous steps' blocks), then the step
    misa.pool_keys(prob, K, ix.Kbar)
    step()
    _status_ok()
    ref_i, ref_v = ix.idx.clone(), ix.val.clone()
    # captured: the same step as one graph, replayed twice
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                                  # warm the side stream
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(2):
        ix.idx.fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        _status_ok()
        a = torch.sort(ix.idx, dim=1).values
        b = torch.sort(ref_i, dim=1).values
        assert torch.equal(a, b)
        assert torch.equal(torch.sort(ix.val, dim=1).values, torch.sort(ref_v, dim=1).values)
