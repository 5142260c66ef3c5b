"""CUDA path vs the CPU oracle, through the C ABI (B200 only).

Small ragged cases compare every output element; the five full-size
workloads run in the launch configuration bench.py times and are checked on
all rows (decode) or on stratified sampled rows (prefill).
"""
import numpy as np
import pytest
import torch

import long_context_sparse_misa_b200 as misa
import oracle
from misa_synth import make_config, make_workload
from tests import parity

pytestmark = pytest.mark.gpu


def dev(wl):
    prob = misa.Problem.from_workload(wl)
    K = torch.from_numpy(wl.K_bits).cuda()
    q = torch.from_numpy(wl.q_bits).cuda()
    w = torch.from_numpy(wl.w).cuda()
    return prob, K, q, w


def status_ok():
    code, bits = misa.stream_status()
    assert code == 0 and bits == 0, f"device status {code} bits {bits}: {misa.lib.misa_last_error_string()}"


def ragged(seed=0, H=16, B=64, m=4, k=100, k_cand=0):
    # several tiles, ragged tails, positions at and around block / tile / k edges
    lens = [700, 1, 300, 129]
    pos = [[0, 1, 62, 63, 64, 99, 100, 101, 127, 128, 255, 256, 511, 640, 699],
           [0], [5, 63, 64, 200, 299], [127, 128]]
    return make_workload(seq_lens=lens, queries=pos, H=H, B=B, m=m, k=k, k_cand=k_cand,
                         seed=seed, name="ragged")


# ------------------------------------------------------------------ pooling
@pytest.mark.parametrize("B", [1, 7, 64, 128, 1000])
def test_pool_keys_bit_exact(B):
    wl = make_workload(seq_lens=[1000, 4133, 63, 1], queries=[[0], [0], [0], [0]], H=4, B=B,
                       seed=3)
    prob, K, q, w = dev(wl)
    Kbar = torch.empty((prob.total_blocks, 128), dtype=torch.float32, device="cuda")
    misa.pool_keys(prob, K, Kbar)
    status_ok()
    ref = oracle.pool_keys(oracle.widen_bf16(wl.K_bits), wl.key_offsets, B)
    np.testing.assert_array_equal(Kbar.cpu().numpy(), ref)
    np.testing.assert_array_equal(prob.block_offsets.cpu().numpy(),
                                  oracle.block_offsets(wl.key_offsets, B))


# ------------------------------------------------------------------ router
# (16, 4, 32), (32, 8, 16), (8, 8, 16) and (64, 1, 32) have enough pooled blocks per
# group to take the split path (tensor-core ranges, finish launch) with 16, 8, 32 and 4
# queries per group; the others run one CTA per group.
@pytest.mark.parametrize("H,m,B", [(16, 4, 64), (64, 8, 64), (32, 8, 128), (8, 8, 16), (64, 1, 32),
                                   (16, 4, 32), (32, 8, 16)])
def test_route_ragged(H, m, B):
    wl = ragged(seed=H + m, H=H, B=B, m=m)
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=m, k=wl.k, with_router_scores=True)
    ix.pool_route(q, w, K)
    status_ok()
    heads = ix.heads.cpu().numpy()
    rep = parity.check_misa_rows(wl, range(wl.T), np.zeros((wl.T, wl.k), np.int32),
                                 np.zeros((wl.T, wl.k), np.float32), heads=heads,
                                 r=ix.r.cpu().numpy(), Kbar=ix.Kbar.cpu().numpy(), m=m,
                                 rep=parity.Report())
    # only the router part of the report matters here
    assert not [f for f in rep.failures if "router" in f or "head" in f or "Kbar" in f], rep.failures
    # compact q_r / w_r are exact gathers of the routed heads
    q_r = ix.q_r.cpu().numpy()
    w_r = ix.w_r.cpu().numpy()
    for i in range(wl.T):
        np.testing.assert_array_equal(q_r[i], wl.q_bits[i][heads[i]])
        np.testing.assert_array_equal(w_r[i], wl.w[i][heads[i]])


# ------------------------------------------------------------------ routed scoring + top-k
@pytest.mark.parametrize("H,m,k", [(16, 4, 100), (64, 8, 256), (32, 8, 1), (64, 64, 50),
                                   (16, 16, 700), (8, 2, 3)])
def test_misa_ragged_full_rows(H, m, k):
    wl = ragged(seed=7 + k, H=H, m=m, k=k)
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=m, k=k)
    L = int(wl.seq_lens.max())
    dbg = torch.full((wl.T, L), float("nan"), dtype=torch.float32, device="cuda")
    ix.misa(q, w, K, scores_dbg=dbg)
    status_ok()
    heads = ix.heads.cpu().numpy()
    rep = parity.check_misa_rows(wl, range(wl.T), ix.idx.cpu().numpy(), ix.val.cpu().numpy(),
                                 heads=heads, k=k, m=m)
    rep.assert_ok()
    # every element of every score row against the oracle with the GPU's heads
    I_gpu = dbg.cpu().numpy()
    Kf = oracle.widen_bf16(wl.K_bits)
    for i in range(wl.T):
        s, t = int(wl.q_seq[i]), int(wl.q_pos[i])
        K_seq = Kf[int(wl.key_offsets[s]):int(wl.key_offsets[s + 1])]
        hs = heads[i].astype(np.int64)
        I_o = oracle.token_scores(oracle.widen_bf16(wl.q_bits[i])[hs], wl.w[i][hs].astype(np.float64),
                                  K_seq[:t + 1])
        np.testing.assert_allclose(I_gpu[i, :t + 1], I_o, rtol=parity.RTOL, atol=parity.ATOL)


def test_routing_every_head_equals_dense_kernel():
    wl = ragged(seed=11, H=32, m=32, k=64)
    prob, K, q, w = dev(wl)
    a = misa.Indexer(prob, m=32, k=64)
    a.misa(q, w, K)
    b = misa.Indexer(prob, m=32, k=64)
    b.dense(q, w, K)
    status_ok()
    for i in range(wl.T):
        assert sorted(a.heads[i].tolist()) == list(range(32))
        ia, ib = a.idx[i].cpu().numpy(), b.idx[i].cpu().numpy()
        assert set(ia.tolist()) == set(ib.tolist())
        va = dict(zip(ia.tolist(), a.val[i].cpu().numpy().tolist()))
        vb = dict(zip(ib.tolist(), b.val[i].cpu().numpy().tolist()))
        for t_ in va:
            if t_ < 0:
                continue  # padding
            assert abs(va[t_] - vb[t_]) <= parity.ATOL + parity.RTOL * abs(vb[t_])
    rep = parity.check_dense_rows(wl, range(wl.T), b.idx.cpu().numpy(), b.val.cpu().numpy())
    rep.assert_ok()


@pytest.mark.parametrize("H,k", [(64, 50), (32, 200), (16, 1)])
def test_dense_ragged(H, k):
    wl = ragged(seed=21 + H, H=H, m=H, k=k)
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=1, k=k)
    ix.dense(q, w, K)
    status_ok()
    parity.check_dense_rows(wl, range(wl.T), ix.idx.cpu().numpy(), ix.val.cpu().numpy()).assert_ok()


def test_empty_sequence_between_others():
    # A sequence with no keys (and so no queries) between two others: its
    # zero blocks and zero rows change nothing for its neighbours.
    wl = make_workload(seq_lens=[500, 0, 300], queries=[[10, 63, 64, 499], [], [0, 127, 299]],
                       H=16, B=64, m=4, k=32, seed=3)
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=wl.m, k=wl.k)
    ix.misa(q, w, K)
    status_ok()
    parity.check_misa_rows(wl, range(wl.T), ix.idx.cpu().numpy(), ix.val.cpu().numpy(),
                           heads=ix.heads.cpu().numpy(), Kbar=ix.Kbar.cpu().numpy()).assert_ok()
    ix.dense(q, w, K)
    status_ok()
    parity.check_dense_rows(wl, range(wl.T), ix.idx.cpu().numpy(), ix.val.cpu().numpy()).assert_ok()


def test_no_queries_is_a_no_op():
    # T = 0: routing, scoring and the dense indexer return at once; only the
    # pooling of the keys (which does not depend on the queries) runs.
    wl = make_workload(seq_lens=[300], queries=[[]], H=8, B=16, m=2, k=4, seed=1)
    assert wl.T == 0
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=wl.m, k=wl.k)
    misa.profile_enable(True)
    ix.misa(q, w, K)
    ix.dense(q, w, K)
    prof = misa.profile_collect()
    misa.profile_enable(False)
    status_ok()
    assert set(prof) <= {"pool_keys"}, prof
    assert ix.idx.shape == (0, wl.k)
    Kbar_o = oracle.pool_keys(oracle.widen_bf16(wl.K_bits), wl.key_offsets, wl.B)
    np.testing.assert_array_equal(ix.Kbar.cpu().numpy(), Kbar_o.astype(np.float32))


def test_hier_whole_prefix_is_dense():
    wl = ragged(seed=31, H=64, m=8, k=40, k_cand=1024)
    prob, K, q, w = dev(wl)
    h = misa.Indexer(prob, m=8, k=40, k_cand=1024)
    h.hier(q, w, K)
    d = misa.Indexer(prob, m=8, k=40)
    d.dense(q, w, K)
    status_ok()
    for i in range(wl.T):
        assert set(h.idx[i].tolist()) == set(d.idx[i].tolist())
    parity.check_rerank_rows(wl, range(wl.T), h.cand.cpu().numpy(), h.idx.cpu().numpy(),
                             h.val.cpu().numpy()).assert_ok()


def test_hier_ragged_candidates():
    wl = ragged(seed=41, H=32, m=4, k=30, k_cand=200)
    prob, K, q, w = dev(wl)
    h = misa.Indexer(prob, m=4, k=30, k_cand=200)
    h.hier(q, w, K)
    status_ok()
    # coarse pass is MISA with k = k_cand; fine pass re-ranks the GPU's own candidates
    parity.check_misa_rows(wl, range(wl.T), h.cand.cpu().numpy(), h.cand_val.cpu().numpy(),
                           heads=h.heads.cpu().numpy(), k=200, m=4).assert_ok()
    parity.check_rerank_rows(wl, range(wl.T), h.cand.cpu().numpy(), h.idx.cpu().numpy(),
                             h.val.cpu().numpy(), k=30).assert_ok()


def test_rerank_skips_padding_and_flags_future_candidates():
    wl = make_workload(seq_lens=[300], queries=[[150]], H=16, B=64, m=4, k=4, seed=5)
    prob, K, q, w = dev(wl)
    cand = torch.tensor([[3, -1, 140, 150, 7, -1, 9, 100]], dtype=torch.int32, device="cuda")
    ix = misa.Indexer(prob, m=4, k=4, k_cand=8)
    misa.hier_rerank(prob, q, w, K, cand, 8, 4, ix.idx, ix.val, ix.ws)
    status_ok()
    parity.check_rerank_rows(wl, [0], cand.cpu().numpy(), ix.idx.cpu().numpy(),
                             ix.val.cpu().numpy(), k=4).assert_ok()
    bad = torch.tensor([[3, 200, 140, 150, 7, -1, 9, 100]], dtype=torch.int32, device="cuda")
    misa.hier_rerank(prob, q, w, K, bad, 8, 4, ix.idx, ix.val, ix.ws)
    code, bits = misa.stream_status()
    assert bits & 0x4 and code == 7
    assert 200 not in ix.idx[0].tolist()


# ------------------------------------------------------------------ status / errors
def test_timeout_selftest_leaves_context_usable():
    misa.selftest_timeout(50)
    code, bits = misa.stream_status()
    assert code == 5 and bits == 1
    code, bits = misa.stream_status()
    assert code == 0 and bits == 0
    test_pool_keys_bit_exact(64)


def test_bad_position_is_flagged_and_row_padded():
    wl = make_workload(seq_lens=[100], queries=[[10, 50]], H=8, B=16, m=2, k=5, seed=1)
    wl.q_pos[1] = 100  # outside the sequence
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=2, k=5)
    ix.misa(q, w, K)
    code, bits = misa.stream_status()
    assert bits & 0x4
    assert ix.idx[1].tolist() == [-1] * 5
    assert len(set(ix.idx[0].tolist())) == 5


# ------------------------------------------------------------------ the five workloads
def _stratified_rows(wl, n):
    T = wl.T
    rows = set(np.linspace(0, T - 1, n // 2).astype(int).tolist())
    rng = np.random.default_rng(0)
    rows |= set(rng.choice(T, n - len(rows), replace=False).tolist())
    rows |= {0, 1, wl.B - 1, wl.B, 127, 128, wl.k - 1, wl.k, wl.k + 1, T - 1}
    return sorted(r for r in rows if 0 <= r < T)


@pytest.mark.parametrize("cfg", [0, 1])
def test_config_decode_all_rows(cfg):
    wl = make_config(cfg)
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=wl.m, k=wl.k, with_router_scores=True)
    ix.misa(q, w, K)
    d = misa.Indexer(prob, m=wl.m, k=wl.k)
    d.dense(q, w, K)
    status_ok()
    rep = parity.check_misa_rows(wl, range(wl.T), ix.idx.cpu().numpy(), ix.val.cpu().numpy(),
                                 heads=ix.heads.cpu().numpy(), r=ix.r.cpu().numpy(),
                                 Kbar=ix.Kbar.cpu().numpy())
    rep.assert_ok()
    parity.check_dense_rows(wl, range(wl.T), d.idx.cpu().numpy(), d.val.cpu().numpy()).assert_ok()
    print(f"config {cfg}: rows={rep.rows} head_swaps={rep.head_swaps} topk_swaps={rep.topk_swaps}")


def test_config0_m_equals_H_is_dense():
    wl = make_config(0)
    prob, K, q, w = dev(wl)
    a = misa.Indexer(prob, m=64, k=wl.k)
    a.misa(q, w, K)
    b = misa.Indexer(prob, m=64, k=wl.k)
    b.dense(q, w, K)
    status_ok()
    for i in range(wl.T):
        assert set(a.idx[i].tolist()) == set(b.idx[i].tolist())


def test_config4_hier_all_rows():
    wl = make_config(4)
    prob, K, q, w = dev(wl)
    h = misa.Indexer(prob, m=wl.m, k=wl.k, k_cand=wl.k_cand)
    h.hier(q, w, K)
    d = misa.Indexer(prob, m=wl.m, k=wl.k)
    d.dense(q, w, K)
    status_ok()
    rows = range(wl.T)
    parity.check_misa_rows(wl, rows, h.cand.cpu().numpy(), h.cand_val.cpu().numpy(),
                           heads=h.heads.cpu().numpy(), k=wl.k_cand).assert_ok()
    parity.check_rerank_rows(wl, rows, h.cand.cpu().numpy(), h.idx.cpu().numpy(),
                             h.val.cpu().numpy()).assert_ok()
    parity.check_dense_rows(wl, rows, d.idx.cpu().numpy(), d.val.cpu().numpy()).assert_ok()
    rec = [oracle.recall_iou(h.idx[i].cpu().numpy(), d.idx[i].cpu().numpy()) for i in rows]
    print("hier recall/IoU vs dense:", np.mean([r[0] for r in rec]), np.mean([r[1] for r in rec]))


def _prefill_invariants(wl, idx):
    """Every row: causal, distinct, min(k, n) entries."""
    n = torch.from_numpy(wl.q_pos.astype(np.int64) + 1).cuda()
    valid = idx >= 0
    assert torch.equal(valid.sum(1), torch.clamp(n, max=wl.k))
    assert bool((idx <= (n - 1)[:, None]).all())
    srt = torch.sort(idx, dim=1).values
    dup = (srt[:, 1:] == srt[:, :-1]) & (srt[:, 1:] >= 0)
    assert not bool(dup.any())


@pytest.mark.parametrize("cfg", [2, 3])
def test_config_prefill_sampled_rows(cfg):
    wl = make_config(cfg)
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=wl.m, k=wl.k)
    misa.profile_enable(True)
    ix.misa(q, w, K)
    prof = misa.profile_collect()
    misa.profile_enable(False)
    status_ok()
    rows = _stratified_rows(wl, 256)
    sel = torch.tensor(rows, device="cuda")
    rep = parity.check_misa_rows(wl, rows, ix.idx[sel].cpu().numpy(), ix.val[sel].cpu().numpy(),
                                 heads=ix.heads[sel].cpu().numpy())
    rep.assert_ok()
    _prefill_invariants(wl, ix.idx)
    rescans = prof.get("#rescan_queries", (0.0, 0))[1]
    print(f"config {cfg}: sampled rows={rep.rows} head_swaps={rep.head_swaps} "
          f"topk_swaps={rep.topk_swaps} rescanned queries={rescans}")
    assert rescans <= wl.T // 100


@pytest.mark.parametrize("cfg", [2, 3])
def test_config_prefill_dense_sampled_rows(cfg):
    """The dense DSA indexer at the full prefill sizes, in the launch
    configuration bench.py times (the same Indexer call)."""
    wl = make_config(cfg)
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=wl.m, k=wl.k)
    misa.profile_enable(True)
    ix.dense(q, w, K)
    prof = misa.profile_collect()
    misa.profile_enable(False)
    status_ok()
    assert "topk" not in prof and "score" in prof and "select" in prof
    rows = _stratified_rows(wl, 256)
    sel = torch.tensor(rows, device="cuda")
    rep = parity.check_dense_rows(wl, rows, ix.idx[sel].cpu().numpy(), ix.val[sel].cpu().numpy())
    rep.assert_ok()
    _prefill_invariants(wl, ix.idx)
    rescans = prof.get("#rescan_queries", (0.0, 0))[1]
    print(f"config {cfg} dense: sampled rows={rep.rows} topk_swaps={rep.topk_swaps} "
          f"rescanned queries={rescans}")
    # the sampled threshold holds for all but a few queries
    assert rescans <= wl.T // 100


# ------------------------------------------------------------------ NaN inputs
NAN_BF16 = np.uint16(0x7FC0)


def test_nan_router_score_ranks_the_head_last_and_is_flagged():
    wl = ragged(seed=51, H=16, m=4, k=60)
    wl.q_bits[3, 5, 17] = NAN_BF16          # one element of head 5 of query row 3
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=4, k=60)
    ix.misa(q, w, K)
    code, bits = misa.stream_status()
    assert bits & 0x4 and code == 7
    heads = ix.heads.cpu().numpy()
    assert 5 not in heads[3].tolist()
    # every row (the NaN head left out of row 3) against the oracle, whose
    # router also ranks the NaN score last
    parity.check_misa_rows(wl, range(wl.T), ix.idx.cpu().numpy(), ix.val.cpu().numpy(),
                           heads=heads, m=4).assert_ok()
    status_ok()


@pytest.mark.parametrize("streamed", [False, True])
def test_nan_token_scores_fill_only_short_rows_and_are_flagged(streamed):
    if streamed:
        wl = make_workload(seq_lens=[10000], queries="all", H=8, B=64, m=8, k=64, seed=52)
        bad = 7000
    else:
        wl = ragged(seed=52, H=8, m=8, k=60)
        bad = 9                               # position 128 of the first sequence
    wl.w[bad, :] = np.nan                     # every head of one query: all its scores NaN
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=8, k=wl.k)
    ix.dense(q, w, K)
    code, bits = misa.stream_status()
    assert bits & 0x4 and code == 7
    idx, val = ix.idx.cpu().numpy(), ix.val.cpu().numpy()
    n = int(wl.q_pos[bad]) + 1
    kk = min(wl.k, n)
    # no numbers in the row: the first min(k, n) tokens (ties go to the lower index), value NaN
    assert sorted(idx[bad][idx[bad] >= 0].tolist()) == list(range(kk))
    assert np.isnan(val[bad][:kk]).all() if not streamed else np.isnan(val[bad][idx[bad] >= 0]).all()
    rows = [i for i in (list(range(wl.T)) if not streamed else [0, 2047, 5000, 6999, 7001, 9999])
            if i != bad]
    parity.check_dense_rows(wl, rows, idx[rows], val[rows]).assert_ok()
    status_ok()
