"""Routed heads x block pruning on the GPU (B200 only), through the C ABI.

The heads the router keeps score the pooled blocks, the best blocks' tokens
(plus the query's own incomplete block) are scored by the same heads and the
top-k is kept (HISA abstract on the thelatestinai.com papers page; MISA
paper, gist.science summary, "Betekenis en Claims").  Checked against the
CPU oracle row by row: heads, kept blocks (near-threshold swaps allowed and
counted), then the top-k over the candidates the GPU's blocks give.
"""
import numpy as np
import pytest
import torch

import long_context_sparse_misa_b200 as misa
from misa_synth import make_config, make_workload
from tests import parity
from tests.test_gpu_parity import dev, ragged, status_ok

pytestmark = pytest.mark.gpu


def run_blocks(wl, nb, m=None, k=None):
    m = wl.m if m is None else m
    k = wl.k if k is None else k
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=m, k=k, n_blocks=nb)
    ix.blocks(q, w, K)
    status_ok()
    return ix


def check(wl, ix, nb, rows=None, m=None, k=None):
    rows = range(wl.T) if rows is None else rows
    sel = list(rows)
    rep = parity.check_block_rows(wl, sel, ix.heads.cpu().numpy()[sel],
                                  ix.blocks_kept.cpu().numpy()[sel], ix.idx.cpu().numpy()[sel],
                                  ix.val.cpu().numpy()[sel], nb, k=k, m=m)
    rep.assert_ok()
    assert rep.rows == len(sel)
    return rep


@pytest.mark.parametrize("H,m,B,k,nb", [(16, 4, 64, 100, 3), (16, 4, 64, 100, 1),
                                        (64, 8, 32, 40, 6), (32, 16, 128, 300, 2)])
def test_blocks_ragged(H, m, B, k, nb):
    # positions below one block (only the incomplete block), at block and
    # tile edges, and past the first k keys; one sequence of a single key
    wl = ragged(seed=H + nb, H=H, B=B, m=m, k=k)
    ix = run_blocks(wl, nb)
    check(wl, ix, nb)


def test_blocks_keeping_every_block_is_misa():
    wl = ragged(seed=77, H=16, B=64, m=4, k=100)
    nb = 700 // 64 + 1
    ix = run_blocks(wl, nb)
    check(wl, ix, nb)
    prob, K, q, w = dev(wl)
    ref = misa.Indexer(prob, m=4, k=100)
    ref.misa(q, w, K)
    status_ok()
    for i in range(wl.T):
        assert set(ix.idx[i].tolist()) == set(ref.idx[i].tolist()), i


def test_blocks_of_one_key_keep_the_routed_topk():
    # B = 1: a pooled block is its key, so the k best blocks are MISA's top-k
    wl = make_workload(seq_lens=[700, 300], queries=[[0, 40, 63, 699], [5, 200, 299]], H=16,
                       B=1, m=4, k=50, seed=12)
    ix = run_blocks(wl, 50)
    check(wl, ix, 50)


@pytest.mark.parametrize("cfg", [0, 1, 4])
def test_blocks_decode_workloads(cfg):
    # the decode workloads with 2k/B kept blocks (candidates: twice the top-k
    # budget plus the incomplete block), every row
    wl = make_config(cfg)
    nb = 2 * wl.k // wl.B
    ix = run_blocks(wl, nb)
    check(wl, ix, nb)


def test_blocks_decode_step_in_cuda_graph_equals_eager():
    wl = make_config(1)
    nb = 2 * wl.k // wl.B
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=wl.m, k=wl.k, n_blocks=nb)
    new_from = torch.tensor(wl.seq_lens - np.diff(wl.query_offsets), dtype=torch.int32,
                            device="cuda")
    misa.pool_keys(prob, K, ix.Kbar)
    step = lambda: ix.blocks(q, w, K, pool_from=new_from)
    step()
    status_ok()
    ref_i, ref_v = ix.idx.clone(), ix.val.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    ix.idx.fill_(-7)
    g.replay()
    torch.cuda.synchronize()
    status_ok()
    # row order is unspecified (the top-k writes its slots in arrival order):
    # compare each row's sorted indices and sorted values
    assert torch.equal(torch.sort(ix.idx, dim=1).values, torch.sort(ref_i, dim=1).values)
    assert torch.equal(torch.sort(ix.val, dim=1).values, torch.sort(ref_v, dim=1).values)
