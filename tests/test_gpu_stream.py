"""The streaming scorer (top-k fused into the tcgen05 epilogue) vs the
materialised-rows path and the CPU oracle, through the C ABI (B200 only).

The streaming path is chosen by the library when there are enough query
groups to fill the GPU (here: prefills of about 10K queries); passing a
scores_dbg buffer forces the materialised path on the same inputs.  Both
compute bit-identical scores, so their selections must be identical.
"""
import dataclasses

import numpy as np
import pytest
import torch

import long_context_sparse_misa_b200 as misa
import oracle
from misa_synth import f32_to_bf16_bits, make_workload
from tests import parity

pytestmark = pytest.mark.gpu


def dev(wl):
    prob = misa.Problem.from_workload(wl)
    return (prob, torch.from_numpy(wl.K_bits).cuda(), torch.from_numpy(wl.q_bits).cuda(),
            torch.from_numpy(wl.w).cuda())


def status_ok():
    code, bits = misa.stream_status()
    assert code == 0 and bits == 0, f"device status {code}/{bits}"


def run_both(wl, dense=False):
    """(stream idx, stream val, rows idx, rows val, heads) for one workload."""
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=wl.m, k=wl.k)
    L = int(wl.seq_lens.max())
    dbg = torch.empty((wl.T, L), dtype=torch.float32, device="cuda")
    misa.profile_enable(True)
    if dense:
        ix.dense(q, w, K)
    else:
        ix.misa(q, w, K)
    prof = misa.profile_collect()
    misa.profile_enable(False)
    status_ok()
    si, sv = ix.idx.clone(), ix.val.clone()
    if dense:
        ix.dense(q, w, K, scores_dbg=dbg)
    else:
        misa.score_topk(prob, ix.q_r, ix.w_r, wl.m, K, wl.k, ix.idx, ix.val, ix.ws, dbg)
    status_ok()
    assert "topk" not in prof, "streaming path was not taken"
    return si, sv, ix.idx, ix.val, ix.heads


def same_sets(si, sv, ri, rv):
    a, b = torch.sort(si, dim=1), torch.sort(ri, dim=1)
    assert torch.equal(a.values, b.values), "selections differ"
    va = torch.gather(sv, 1, a.indices)
    vb = torch.gather(rv, 1, b.indices)
    assert torch.equal(va, vb), "values differ"


def invariants(wl, idx):
    n = torch.from_numpy(wl.q_pos.astype(np.int64) + 1).cuda()
    valid = idx >= 0
    assert torch.equal(valid.sum(1), torch.clamp(n, max=wl.k))
    assert bool((idx <= (n - 1)[:, None]).all())
    srt = torch.sort(idx, dim=1).values
    assert not bool(((srt[:, 1:] == srt[:, :-1]) & (srt[:, 1:] >= 0)).any())


def sample_rows(wl, n=80):
    rng = np.random.default_rng(1)
    rows = set(rng.choice(wl.T, n, replace=False).tolist())
    rows |= {0, 1, wl.k - 1, wl.k, wl.k + 1, wl.T - 1}
    return sorted(r for r in rows if r < wl.T)


@pytest.mark.parametrize("H,m,B,k", [(32, 8, 128, 256), (64, 8, 64, 2048), (32, 16, 128, 100),
                                     (64, 8, 64, 1)])
def test_stream_matches_rows_and_oracle(H, m, B, k):
    wl = make_workload(seq_lens=[10000], queries="all", H=H, B=B, m=m, k=k, seed=H + k)
    si, sv, ri, rv, heads = run_both(wl)
    same_sets(si, sv, ri, rv)
    invariants(wl, si)
    rows = sample_rows(wl)
    sel = torch.tensor(rows, device="cuda")
    parity.check_misa_rows(wl, rows, si[sel].cpu().numpy(), sv[sel].cpu().numpy(),
                           heads=heads[sel].cpu().numpy(), k=k, m=m).assert_ok()


def test_stream_selection_after_the_pass_and_in_kernel_agree():
    # The workspace misa_workspace_size reports holds candidate lists per query,
    # selected by a launch after the scoring pass; a smaller one (down to the
    # double-buffered lists) selects inside the scoring kernel.  Same top-k.
    wl = make_workload(seq_lens=[10000], queries="all", H=32, B=128, m=8, k=512, seed=31)
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=wl.m, k=wl.k)
    misa.profile_enable(True)
    ix.misa(q, w, K)
    prof = misa.profile_collect()
    misa.profile_enable(False)
    status_ok()
    assert "select" in prof and "topk" not in prof
    di, dv = ix.idx.clone(), ix.val.clone()
    small = ix.ws[: ix.ws.numel() - 256]
    misa.profile_enable(True)
    misa.score_topk(prob, ix.q_r, ix.w_r, wl.m, K, wl.k, ix.idx, ix.val, small)
    prof = misa.profile_collect()
    misa.profile_enable(False)
    status_ok()
    assert "select" not in prof and "topk" not in prof and "score" in prof
    same_sets(di, dv, ix.idx, ix.val)
    invariants(wl, di)
    rows = sample_rows(wl, 30)
    sel = torch.tensor(rows, device="cuda")
    parity.check_misa_rows(wl, rows, di[sel].cpu().numpy(), dv[sel].cpu().numpy(),
                           heads=ix.heads[sel].cpu().numpy(), k=wl.k, m=wl.m).assert_ok()


def test_stream_dense_multi_sequence():
    wl = make_workload(seq_lens=[5000, 3000, 2700], queries="all", H=32, B=128, m=8, k=512,
                       seed=9)
    si, sv, ri, rv, _ = run_both(wl, dense=True)
    same_sets(si, sv, ri, rv)
    invariants(wl, si)
    rows = sample_rows(wl, 40)
    sel = torch.tensor(rows, device="cuda")
    parity.check_dense_rows(wl, rows, si[sel].cpu().numpy(), sv[sel].cpu().numpy()).assert_ok()


def test_stream_increasing_scores_every_key_appended():
    # Scores grow with the key index, so every key beats the running threshold.
    L, H, d = 10000, 8, 128
    wl = make_workload(seq_lens=[L], queries="all", H=H, B=64, m=8, k=300, seed=2,
                       needles=False)
    u = np.zeros(d, np.float32)
    u[:4] = 0.5
    K = (np.arange(1, L + 1, dtype=np.float32)[:, None] / L) * u[None, :]
    q = np.broadcast_to(u, (L, H, d)).astype(np.float32)
    wl = dataclasses.replace(wl, K_bits=f32_to_bf16_bits(K), q_bits=f32_to_bf16_bits(q),
                             w=np.full((L, H), 0.5, np.float32))
    si, sv, ri, rv, heads = run_both(wl)
    same_sets(si, sv, ri, rv)
    invariants(wl, si)
    rows = [0, 299, 300, 5000, L - 1]
    sel = torch.tensor(rows, device="cuda")
    parity.check_misa_rows(wl, rows, si[sel].cpu().numpy(), sv[sel].cpu().numpy(),
                           heads=heads[sel].cpu().numpy()).assert_ok()


def test_stream_exact_ties_resolve_to_lower_index():
    # Keys and queries on a coarse grid: many exactly equal scores, incl. zeros.
    L, H, d = 9600, 8, 128
    rng = np.random.default_rng(4)
    wl = make_workload(seq_lens=[L], queries="all", H=H, B=64, m=8, k=700, seed=3,
                       needles=False)
    K = rng.integers(-1, 2, size=(L, d)).astype(np.float32)
    K[:, 2:] = 0
    q = np.zeros((L, H, d), np.float32)
    q[:, :, :2] = rng.integers(-1, 2, size=(L, H, 2))
    wl = dataclasses.replace(wl, K_bits=f32_to_bf16_bits(K), q_bits=f32_to_bf16_bits(q),
                             w=np.full((L, H), 0.25, np.float32))
    si, sv, ri, rv, heads = run_both(wl)
    same_sets(si, sv, ri, rv)
    invariants(wl, si)
    rows = sample_rows(wl, 30)
    sel = torch.tensor(rows, device="cuda")
    hs = heads[sel].cpu().numpy()
    # exact ties: the selected set must equal the oracle's exactly (no tolerance games)
    Kf = oracle.widen_bf16(wl.K_bits)
    for j, i in enumerate(rows):
        t = int(wl.q_pos[i])
        I = oracle.token_scores(oracle.widen_bf16(wl.q_bits[i])[hs[j]],
                                wl.w[i][hs[j]].astype(np.float64), Kf[:t + 1])
        ref, _ = oracle.topk(I, wl.k)
        assert set(si[i].tolist()) == set(ref.tolist()), f"row {i}"


def test_stream_probe_overestimate_goes_through_fixup():
    # The probed tiles (every 24th, from tile 12) all lie among the tiles that
    # hold high scores (every 8th, from tile 4), on half their keys: the
    # sampled threshold then admits fewer than k keys, the check fails and
    # those queries are rescanned without a probe.
    L, H, d = 10000, 8, 128
    wl = make_workload(seq_lens=[L], queries="all", H=H, B=64, m=8, k=2048, seed=6,
                       needles=False)
    K = np.zeros((L, d), np.float32)
    K[:, 0] = 1.0
    s = np.arange(L)
    high = ((s // 128) % 8 == 4) & (s % 2 == 0)
    K[high, 0] = 10.0
    q = np.zeros((L, H, d), np.float32)
    q[:, :, 0] = 1.0
    wl = dataclasses.replace(wl, K_bits=f32_to_bf16_bits(K), q_bits=f32_to_bf16_bits(q),
                             w=np.full((L, H), 0.125, np.float32))
    prob, Kd, qd, wd = dev(wl)
    ix = misa.Indexer(prob, m=wl.m, k=wl.k)
    misa.profile_enable(True)
    ix.misa(qd, wd, Kd)
    prof = misa.profile_collect()
    misa.profile_enable(False)
    status_ok()
    # the queries with the overestimating sample (long enough to be probed):
    # more than the split rescan takes, so both rescan paths run
    assert prof["#rescan_queries"][1] > 1000
    assert "rescan_score" in prof and "rescan_topk" in prof and "score_fixup" in prof
    si, sv = ix.idx.clone(), ix.val.clone()
    dbg = torch.empty((wl.T, L), dtype=torch.float32, device="cuda")
    misa.score_topk(prob, ix.q_r, ix.w_r, wl.m, Kd, wl.k, ix.idx, ix.val, ix.ws, dbg)
    status_ok()
    same_sets(si, sv, ix.idx, ix.val)
    invariants(wl, si)
    rows = [0, 2047, 2048, 5000, L - 1]
    Kf = oracle.widen_bf16(wl.K_bits)
    for i in rows:
        I = oracle.token_scores(oracle.widen_bf16(wl.q_bits[i])[:8], wl.w[i][:8].astype(np.float64),
                                Kf[:i + 1])
        ref, _ = oracle.topk(I, wl.k)
        assert set(si[i].tolist()) == set(ref.tolist()), f"row {i}"


def test_hier_prefill_streamed_candidates_then_rerank():
    # MISA-dagger in prefill: the coarse keep (k' = 1024) runs on the streaming
    # scorer, then every query re-ranks its candidates with all heads.
    wl = make_workload(seq_lens=[12000], queries="all", H=32, B=128, m=8, k=128, k_cand=1024,
                       seed=21)
    prob, K, q, w = dev(wl)
    ix = misa.Indexer(prob, m=wl.m, k=wl.k, k_cand=wl.k_cand)
    misa.profile_enable(True)
    ix.hier(q, w, K)
    prof = misa.profile_collect()
    misa.profile_enable(False)
    status_ok()
    assert "topk" in prof and "score" in prof  # streamed keep, then the rerank's top-k
    invariants(dataclasses.replace(wl, k=wl.k_cand), ix.cand)
    invariants(wl, ix.idx)
    rows = sample_rows(wl, 40)
    sel = torch.tensor(rows, device="cuda")
    parity.check_misa_rows(wl, rows, ix.cand[sel].cpu().numpy(), ix.cand_val[sel].cpu().numpy(),
                           heads=ix.heads[sel].cpu().numpy(), k=wl.k_cand,
                           m=wl.m).assert_ok()
    parity.check_rerank_rows(wl, rows, ix.cand[sel].cpu().numpy(), ix.idx[sel].cpu().numpy(),
                             ix.val[sel].cpu().numpy()).assert_ok()


def test_stream_dense_rescan_at_prefill_size():
    # The probe-overestimate pattern with all heads (the dense indexer) over a
    # 32K prefill: most queries fail their sampled threshold and go through
    # the rescan launch, which must still give the exact top-k.
    L, H, d = 32768, 32, 128
    wl = make_workload(seq_lens=[L], queries="all", H=H, B=128, m=H, k=2048, seed=8,
                       needles=False)
    K = np.zeros((L, d), np.float32)
    K[:, 0] = 1.0
    s = np.arange(L)
    high = ((s // 128) % 8 == 4) & (s % 2 == 0)
    K[high, 0] = 10.0
    K[:, 1] = (s % 7) * 0.125  # distinct scores inside a tile
    rng = np.random.default_rng(8)
    q = np.zeros((L, H, d), np.float32)
    q[:, :, 0] = 1.0
    q[:, :, 1] = rng.integers(0, 3, size=(L, H)) * 0.5
    w = rng.uniform(0.05, 0.2, size=(L, H)).astype(np.float32)
    wl = dataclasses.replace(wl, K_bits=f32_to_bf16_bits(K), q_bits=f32_to_bf16_bits(q), w=w)
    prob, Kd, qd, wd = dev(wl)
    ix = misa.Indexer(prob, m=8, k=wl.k)
    misa.profile_enable(True)
    ix.dense(qd, wd, Kd)
    prof = misa.profile_collect()
    misa.profile_enable(False)
    status_ok()
    assert "topk" not in prof
    assert prof["#rescan_queries"][1] > L // 4
    invariants(wl, ix.idx)
    rows = [0, 2047, 2048, 2049, 9000, 20000, L - 2, L - 1]
    sel = torch.tensor(rows, device="cuda")
    parity.check_dense_rows(wl, rows, ix.idx[sel].cpu().numpy(),
                            ix.val[sel].cpu().numpy()).assert_ok()


def test_stream_few_failures_rescanned_as_score_rows():
    # Six 1940-key sequences, k = 512: only queries with at least 16 tiles of
    # prefix (positions 1920..1939) are probed, and the probe tile (tile 12)
    # holds the high scores of the overestimate pattern, so about 20 queries
    # per sequence fail: fewer than the split rescan takes (128), which
    # scores them as full rows over several CTAs each and selects from those.
    lens = [1940] * 6
    H, d = 8, 128
    wl = make_workload(seq_lens=lens, queries="all", H=H, B=64, m=8, k=512, seed=12,
                       needles=False)
    L = sum(lens)
    K = np.zeros((L, d), np.float32)
    K[:, 0] = 1.0
    s = np.concatenate([np.arange(n) for n in lens])
    high = ((s // 128) % 8 == 4) & (s % 2 == 0)
    K[high, 0] = 10.0
    K[:, 1] = (s % 5) * 0.25
    q = np.zeros((wl.T, H, d), np.float32)
    q[:, :, 0] = 1.0
    q[:, :, 1] = 0.5
    wl = dataclasses.replace(wl, K_bits=f32_to_bf16_bits(K), q_bits=f32_to_bf16_bits(q),
                             w=np.full((wl.T, H), 0.125, np.float32))
    prob, Kd, qd, wd = dev(wl)
    ix = misa.Indexer(prob, m=wl.m, k=wl.k)
    misa.profile_enable(True)
    ix.misa(qd, wd, Kd)
    prof = misa.profile_collect()
    misa.profile_enable(False)
    status_ok()
    n_fail = prof["#rescan_queries"][1]
    assert 0 < n_fail <= 128, n_fail
    si, sv = ix.idx.clone(), ix.val.clone()
    dbg = torch.empty((wl.T, max(lens)), dtype=torch.float32, device="cuda")
    misa.score_topk(prob, ix.q_r, ix.w_r, wl.m, Kd, wl.k, ix.idx, ix.val, ix.ws, dbg)
    status_ok()
    same_sets(si, sv, ix.idx, ix.val)
    invariants(wl, si)
    rows = [1935, 1939, 1940 + 1925, 5 * 1940 + 1939]
    sel = torch.tensor(rows, device="cuda")
    parity.check_misa_rows(wl, rows, si[sel].cpu().numpy(), sv[sel].cpu().numpy(),
                           heads=ix.heads[sel].cpu().numpy()).assert_ok()
