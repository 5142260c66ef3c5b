"""Pins for the CPU oracle, independent of the oracle's own code.

Each test checks the oracle against something the pages or mathematics fix:
a hand-worked example (tests/golden/worked_tiny.json), closed forms, brute
force written as plain Python loops on tiny inputs, and the identities the
method states (routing every head is the dense DSA indexer; re-ranking the
whole prefix with all heads is DSA top-k).  test_oracle_mutants.py plants
plausible mistakes in the oracle and checks that these pins catch them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from misa_synth import bf16_bits_to_f32, f32_to_bf16_bits, make_workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_tiny.json")


def _f(x):
    return -math.inf if x == "-inf" else float(x)


def load_golden():
    with open(GOLDEN) as f:
        return json.load(f)


# ---------------------------------------------------------------- bf16 widening
def test_widen_bf16_known_patterns():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000, 0x7F80], dtype=np.uint16)
    v = oracle.widen_bf16(bits)
    assert v[0] == 1.0 and v[1] == -2.0 and v[2] == 1.0 + 2.0 ** -7
    assert v[3] == 0.0 and v[4] == 0.0 and math.copysign(1, v[4]) == -1 and v[5] == math.inf


# ---------------------------------------------------------------- hand-worked example
def _golden_arrays(g):
    K = oracle.widen_bf16(f32_to_bf16_bits(np.array(g["K"], dtype=np.float32)))
    Kbar = oracle.pool_keys(K, np.array([0, len(K)]), g["B"])
    return K, Kbar


def test_golden_pooled_keys():
    g = load_golden()
    _, Kbar = _golden_arrays(g)
    np.testing.assert_array_equal(Kbar, np.array(g["Kbar"], dtype=np.float32))


@pytest.mark.parametrize("case", range(6))
def test_golden_case(case):
    g = load_golden()
    c = g["cases"][case]
    K, Kbar = _golden_arrays(g)
    q = oracle.widen_bf16(f32_to_bf16_bits(np.array(c["q"], dtype=np.float32)))
    w = np.array(c["w"], dtype=np.float64)
    res = oracle.misa_query(q, w, K, Kbar, c["t"], g["B"], c["m"], c["k"])
    np.testing.assert_array_equal(res["r"], np.array(c["r"]))
    np.testing.assert_array_equal(res["heads"], np.array(c["heads"]))
    np.testing.assert_array_equal(res["I"], np.array(c["I_routed"], dtype=np.float64))
    np.testing.assert_array_equal(res["idx"], np.array(c["idx"]))
    np.testing.assert_array_equal(res["val"], np.array([_f(x) for x in c["val"]]))
    if "I_dense" in c:
        dn = oracle.dense_query(q, w, K, c["t"], c["k"])
        np.testing.assert_array_equal(dn["I"], np.array(c["I_dense"], dtype=np.float64))
        np.testing.assert_array_equal(dn["idx"], np.array(c["dense_idx"]))
        np.testing.assert_array_equal(dn["val"], np.array(c["dense_val"], dtype=np.float64))
        coarse = oracle.misa_query(q, w, K, Kbar, c["t"], g["B"], c["m"], c["k_cand"])
        assert sorted(coarse["idx"].tolist()) == sorted(c["cand"])
        hr = oracle.hier_rerank_query(q, w, K, coarse["idx"], c["k"])
        np.testing.assert_array_equal(hr["idx"], np.array(c["hier_idx"]))
        np.testing.assert_array_equal(hr["val"], np.array(c["hier_val"], dtype=np.float64))


# ---------------------------------------------------------------- pooling closed forms
def test_pool_constant_blocks():
    rng = np.random.default_rng(1)
    B, L, d = 8, 37, 16
    consts = rng.integers(-64, 64, size=(math.ceil(L / B), d)) / 16.0
    K = np.repeat(consts, B, axis=0)[:L]
    Kbar = oracle.pool_keys(K, np.array([0, L]), B)
    np.testing.assert_array_equal(Kbar, consts.astype(np.float32))


def test_pool_ramp_and_partial_tail():
    # k[s] = s * c: block mean of keys lo..hi-1 is c*(lo+hi-1)/2; the last
    # block holds L mod B keys and is averaged over those only.
    B, L, d = 16, 53, 4
    c = np.array([1.0, -0.5, 0.25, 2.0])
    K = np.arange(L, dtype=np.float64)[:, None] * c
    Kbar = oracle.pool_keys(K, np.array([0, L]), B)
    for b in range(math.ceil(L / B)):
        lo, hi = b * B, min(b * B + B, L)
        np.testing.assert_array_equal(Kbar[b], (c * (lo + hi - 1) / 2.0).astype(np.float32))


def test_pool_two_sequences_offsets():
    B, d = 4, 2
    L = [5, 3]
    K = np.arange(16, dtype=np.float64).reshape(8, 2)
    Kbar = oracle.pool_keys(K, np.array([0, 5, 8]), B)
    assert Kbar.shape == (2 + 1, d)
    np.testing.assert_array_equal(Kbar[0], [3.0, 4.0])   # keys 0..3
    np.testing.assert_array_equal(Kbar[1], [8.0, 9.0])   # key 4 alone
    np.testing.assert_array_equal(Kbar[2], [12.0, 13.0])  # keys 5..7 of sequence 1
    np.testing.assert_array_equal(oracle.block_offsets(np.array([0, 5, 8]), B), [0, 2, 3])


def test_pool_rounds_once_to_fp32():
    # mean of 3 keys 1/3-ish: fp64 mean, one rounding to fp32
    K = np.array([[1.0], [1.0], [2.0 ** -9]])
    Kbar = oracle.pool_keys(K, np.array([0, 3]), 4)
    assert Kbar[0, 0] == np.float32((2.0 + 2.0 ** -9) / 3.0)


# ---------------------------------------------------------------- brute force, tiny
def _brute_router(q, w, K, t, B):
    """Plain loops: per head, sum ReLU(q.mean(block)) over visible blocks."""
    H, d = len(q), len(q[0])
    n = t + 1
    r = []
    for h in range(H):
        total = 0.0
        b = 0
        while b * B < n:
            lo, hi = b * B, min(b * B + B, n)
            if hi - lo == B:   # full block: pooled value rounded to fp32
                mean = [float(np.float32(sum(K[s][j] for s in range(lo, hi)) / (hi - lo)))
                        for j in range(d)]
            else:              # causal partial block, fp64
                mean = [sum(K[s][j] for s in range(lo, hi)) / (hi - lo) for j in range(d)]
            dot = sum(q[h][j] * mean[j] for j in range(d))
            total += dot if dot > 0 else 0.0
            b += 1
        r.append(w[h] * total)
    return r


def _brute_scores(q, w, heads, K, t):
    out = []
    for s in range(t + 1):
        acc = 0.0
        for h in heads:
            dot = sum(q[h][j] * K[s][j] for j in range(len(K[s])))
            acc += w[h] * (dot if dot > 0 else 0.0)
        out.append(acc)
    return out


def _brute_topk(I, k):
    order = sorted(range(len(I)), key=lambda s: (-(I[s] + 0.0), s))[:k]
    return order + [-1] * (k - len(order))


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(100 + seed)
    H = int(rng.integers(1, 7))
    B = int(rng.choice([4, 8]))
    L = int(rng.integers(1, 40))
    d = int(rng.choice([3, 8]))
    m = int(rng.integers(1, H + 1))
    k = int(rng.integers(1, 12))
    K = oracle.widen_bf16(f32_to_bf16_bits(rng.standard_normal((L, d)).astype(np.float32)))
    Kbar = oracle.pool_keys(K, np.array([0, L]), B)
    for t in range(L):
        q = oracle.widen_bf16(f32_to_bf16_bits(rng.standard_normal((H, d)).astype(np.float32)))
        w = rng.standard_normal(H).astype(np.float32).astype(np.float64)
        res = oracle.misa_query(q, w, K, Kbar, t, B, m, k)
        r_ref = _brute_router(q.tolist(), w.tolist(), K.tolist(), t, B)
        np.testing.assert_allclose(res["r"], r_ref, rtol=1e-12, atol=1e-15)
        heads_ref = sorted(range(H), key=lambda h: (-r_ref[h], h))[:m]
        assert res["heads"].tolist() == heads_ref
        I_ref = _brute_scores(q.tolist(), w.tolist(), heads_ref, K.tolist(), t)
        np.testing.assert_allclose(res["I"], I_ref, rtol=1e-12, atol=1e-15)
        assert res["idx"].tolist() == _brute_topk(I_ref, k)


def test_topk_brute_force_with_ties_and_negative_zero():
    I = np.array([0.0, -0.0, 1.5, -1.0, 1.5, 0.0, -0.0, 2.0, -1.0])
    for k in range(1, 12):
        idx, val = oracle.topk(I, k)
        ref = _brute_topk(I.tolist(), k)
        assert idx.tolist() == ref
        for i, v in zip(idx, val):
            if i < 0:
                assert v == -math.inf
            else:
                assert v == I[i] and math.copysign(1.0, v) == 1.0 or v != 0.0


# ---------------------------------------------------------------- special cases
def test_single_block_router_is_dsa_of_mean_key():
    rng = np.random.default_rng(7)
    L, d, H, B = 20, 8, 5, 32
    K = rng.standard_normal((L, d))
    Kbar = oracle.pool_keys(K, np.array([0, L]), B)
    for t in range(L):
        q = rng.standard_normal((H, d))
        w = rng.standard_normal(H)
        mean = K[:t + 1].mean(axis=0)
        expect = w * np.maximum(q @ mean, 0.0)
        np.testing.assert_allclose(oracle.router_scores(q, w, K, Kbar, t, B), expect,
                                   rtol=1e-12, atol=1e-15)


def test_one_head_positive_dots_is_a_matmul():
    # H=1, w=1, all q.k > 0: I reduces to K @ q.
    rng = np.random.default_rng(3)
    K = rng.uniform(0.1, 1.0, size=(50, 16))
    q = rng.uniform(0.1, 1.0, size=(1, 16))
    I = oracle.token_scores(q, np.ones(1), K)
    np.testing.assert_allclose(I, np.matmul(K, q[0]), rtol=1e-14)


def _small_wl(seed=5, H=8, B=8, m=3, k=10):
    return make_workload(seq_lens=[45, 70], queries=[[0, 7, 8, 30, 44], [3, 15, 16, 69]],
                         H=H, d=16, B=B, m=m, k=k, seed=seed, k_cand=25)


def test_routing_every_head_is_dense_dsa():
    wl = _small_wl()
    full = oracle.misa_index(wl, m=wl.H)
    dense = oracle.dense_index(wl)
    for a, b in zip(full["rows"], dense):
        assert sorted(a["heads"].tolist()) == list(range(wl.H))
        np.testing.assert_allclose(a["I"], b["I"], rtol=1e-13, atol=1e-16)
        np.testing.assert_array_equal(a["idx"], b["idx"])


def test_hier_with_whole_prefix_is_dsa_topk():
    wl = _small_wl()
    L = int(np.max(wl.seq_lens))
    hier = oracle.hier_index(wl, k_cand=L)
    dense = oracle.dense_index(wl)
    for a, b in zip(hier, dense):
        np.testing.assert_array_equal(a["idx"], b["idx"])
        np.testing.assert_allclose(a["val"], b["val"], rtol=1e-13)


def test_causality_future_keys_do_not_matter():
    wl = _small_wl()
    base = oracle.misa_index(wl)
    K2 = wl.K_bits.copy()
    # scramble keys after each sequence's earliest query position... per query check
    for i in range(wl.T):
        s = int(wl.q_seq[i])
        t = int(wl.q_pos[i])
        k0, k1 = int(wl.key_offsets[s]), int(wl.key_offsets[s + 1])
        K2 = wl.K_bits.copy()
        K2[k0 + t + 1:k1] = f32_to_bf16_bits(np.full((k1 - k0 - t - 1, wl.d), 3.0, np.float32))
        import dataclasses
        wl2 = dataclasses.replace(wl, K_bits=K2)
        row = oracle.misa_index(wl2, rows=[i])["rows"][0]
        np.testing.assert_array_equal(row["r"], base["rows"][i]["r"])
        np.testing.assert_array_equal(row["idx"], base["rows"][i]["idx"])


def test_dense_head_permutation_invariance():
    wl = _small_wl()
    perm = np.random.default_rng(0).permutation(wl.H)
    import dataclasses
    wl2 = dataclasses.replace(wl, q_bits=wl.q_bits[:, perm], w=wl.w[:, perm])
    for a, b in zip(oracle.dense_index(wl), oracle.dense_index(wl2)):
        np.testing.assert_array_equal(a["idx"], b["idx"])
        np.testing.assert_allclose(a["I"], b["I"], rtol=1e-13)


def test_selection_invariants():
    wl = _small_wl(k=12)
    for i, row in enumerate(oracle.misa_index(wl)["rows"]):
        t = int(wl.q_pos[i])
        sel = [x for x in row["idx"].tolist() if x >= 0]
        assert len(sel) == min(wl.k, t + 1) == len(set(sel))
        assert all(0 <= x <= t for x in sel)
        rest = np.setdiff1d(np.arange(t + 1), sel)
        if len(rest):
            assert row["I"][sel].min() >= row["I"][rest].max()


def test_recall_iou_closed_form():
    assert oracle.recall_iou([1, 2, 3], [2, 3, 4, 5]) == (0.5, 0.4)
    assert oracle.recall_iou([1, 2, -1], [1, 2]) == (1.0, 1.0)
    assert oracle.recall_iou([7], [8]) == (0.0, 0.0)
    assert oracle.recall_iou([], []) == (1.0, 1.0)


# ---------------------------------------------------------------- the generator
def test_bf16_rounding_ties_to_even():
    x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -(1.0 + 2 ** -8)], np.float32)
    np.testing.assert_array_equal(bf16_bits_to_f32(f32_to_bf16_bits(x)),
                                  np.array([1.0, 1.0 + 2 ** -6, 1.0, -1.0], np.float32))


def test_generator_deterministic_and_shaped():
    a = make_workload(seq_lens=[300, 200], queries=3, H=4, d=16, B=8, seed=11)
    b = make_workload(seq_lens=[300, 200], queries=3, H=4, d=16, B=8, seed=11)
    np.testing.assert_array_equal(a.K_bits, b.K_bits)
    np.testing.assert_array_equal(a.q_bits, b.q_bits)
    assert a.K_bits.shape == (500, 16) and a.q_bits.shape == (6, 4, 16) and a.w.shape == (6, 4)
    assert a.q_pos.tolist() == [297, 298, 299, 197, 198, 199]
    assert a.query_offsets.tolist() == [0, 3, 6] and a.pairs == 298 + 299 + 300 + 198 + 199 + 200
    # needles: 1% of keys carry an extra 2*u_h; their norms stand out
    plain = make_workload(seq_lens=[300, 200], queries=3, H=4, d=16, B=8, seed=11,
                          needles=False)
    moved = np.any(plain.K_bits != a.K_bits, axis=1)
    assert moved.sum() == 3 + 2


# ---------------------------------------------------------------- block pruning (head axis x token axis)
BLOCK_GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "block_pruned_tiny.json")


@pytest.mark.parametrize("case", range(4))
def test_block_golden_case(case):
    with open(BLOCK_GOLDEN) as f:
        g = json.load(f)
    c = g["cases"][case]
    K = oracle.widen_bf16(f32_to_bf16_bits(np.array(g["K"], dtype=np.float32)))
    Kbar = oracle.pool_keys(K, np.array([0, len(K)]), g["B"])
    np.testing.assert_array_equal(Kbar, np.array(g["Kbar"], dtype=np.float32))
    q = oracle.widen_bf16(f32_to_bf16_bits(np.array(c["q"], dtype=np.float32)))
    w = np.array(c["w"], dtype=np.float64)
    res = oracle.block_pruned_query(q, w, K, Kbar, c["t"], g["B"], c["m"], c["nb"], c["k"])
    assert res["heads"].tolist() == c["heads"]
    np.testing.assert_array_equal(res["S"], np.array(c["S"], dtype=np.float64))
    assert res["blocks"].tolist() == c["blocks"]
    assert res["cand"].tolist() == c["cand"]
    assert res["idx"].tolist() == c["idx"]
    np.testing.assert_array_equal(res["val"], np.array(c["val"], dtype=np.float64))


@pytest.mark.parametrize("seed", range(4))
def test_block_brute_force_tiny(seed):
    """Plain loops: block scores of the routed heads on the pooled keys, the
    nb best full blocks plus the incomplete block, token top-k inside."""
    rng = np.random.default_rng(300 + seed)
    H = int(rng.integers(1, 7))
    B = int(rng.choice([2, 4, 8]))
    L = int(rng.integers(1, 40))
    d = int(rng.choice([3, 8]))
    m = int(rng.integers(1, H + 1))
    nb = int(rng.integers(1, 4))
    k = int(rng.integers(1, 12))
    K = oracle.widen_bf16(f32_to_bf16_bits(rng.standard_normal((L, d)).astype(np.float32)))
    Kbar = oracle.pool_keys(K, np.array([0, L]), B)
    Kl = K.tolist()
    for t in range(L):
        q = oracle.widen_bf16(f32_to_bf16_bits(rng.standard_normal((H, d)).astype(np.float32)))
        w = rng.standard_normal(H).astype(np.float32).astype(np.float64)
        res = oracle.block_pruned_query(q, w, K, Kbar, t, B, m, nb, k)
        r_ref = _brute_router(q.tolist(), w.tolist(), Kl, t, B)
        heads = sorted(range(H), key=lambda h: (-r_ref[h], h))[:m]
        assert res["heads"].tolist() == heads
        full = (t + 1) // B
        S = []
        for b in range(full):
            mean = [float(np.float32(sum(Kl[s][j] for s in range(b * B, b * B + B)) / B))
                    for j in range(d)]
            acc = 0.0
            for h in heads:
                dot = sum(q[h][j] * mean[j] for j in range(d))
                acc += w[h] * (dot if dot > 0 else 0.0)
            S.append(acc)
        np.testing.assert_allclose(res["S"], S, rtol=1e-12, atol=1e-15)
        kept = sorted(range(full), key=lambda b: (-(S[b] + 0.0), b))[:nb]
        assert res["blocks"].tolist() == kept + [-1] * (nb - len(kept))
        cand = sorted([b * B + j for b in kept for j in range(B)] + list(range(full * B, t + 1)))
        assert res["cand"].tolist() == cand
        I_all = _brute_scores(q.tolist(), w.tolist(), heads, Kl, t)
        order = sorted(cand, key=lambda s: (-(I_all[s] + 0.0), s))[:k]
        assert res["idx"].tolist() == order + [-1] * (k - len(order))
        np.testing.assert_allclose(res["val"][:len(order)], [I_all[s] for s in order],
                                   rtol=1e-12, atol=1e-15)


def test_block_pruning_keeping_every_block_is_routed_topk():
    """Identity: with every full block kept the candidates are the whole
    prefix, so the result is MISA's routed top-k."""
    wl = _small_wl()
    L = int(np.max(wl.seq_lens))
    pruned = oracle.block_index(wl, nb=L)
    misa = oracle.misa_index(wl)["rows"]
    for a, b in zip(pruned, misa):
        np.testing.assert_array_equal(a["heads"], b["heads"])
        np.testing.assert_array_equal(a["idx"], b["idx"])
        np.testing.assert_allclose(a["val"], b["val"], rtol=1e-13)


def test_block_pruning_with_one_key_blocks_is_routed_topk():
    """Special case B = 1: a pooled block is its key (bf16 -> fp32 exact), the
    block score is the token score, so keeping the k best blocks keeps MISA's
    routed top-k tokens."""
    wl = make_workload(seq_lens=[45, 70], queries=[[0, 7, 8, 30, 44], [3, 15, 16, 69]],
                       H=8, d=16, B=1, m=3, k=10, seed=9, k_cand=25)
    pruned = oracle.block_index(wl, nb=wl.k)
    misa = oracle.misa_index(wl)["rows"]
    for a, b in zip(pruned, misa):
        np.testing.assert_array_equal(a["idx"], b["idx"])
        np.testing.assert_allclose(a["val"], b["val"], rtol=1e-13)
        assert sorted(x for x in a["blocks"].tolist() if x >= 0) == \
            sorted(x for x in b["idx"].tolist() if x >= 0)


def test_block_pruning_causality_and_growing_block_budget():
    """Keys after the query's position change nothing (their pooled block is
    never scored, the incomplete block stops at the query); and keeping more
    blocks only adds candidates, so the kept top-k score never drops."""
    import dataclasses
    wl = _small_wl()
    base = oracle.block_index(wl, nb=2)
    for i in range(wl.T):
        s = int(wl.q_seq[i])
        t = int(wl.q_pos[i])
        k0, k1 = int(wl.key_offsets[s]), int(wl.key_offsets[s + 1])
        K2 = wl.K_bits.copy()
        K2[k0 + t + 1:k1] = f32_to_bf16_bits(np.full((k1 - k0 - t - 1, wl.d), 3.0, np.float32))
        row = oracle.block_index(dataclasses.replace(wl, K_bits=K2), nb=2, rows=[i])[0]
        np.testing.assert_array_equal(row["S"], base[i]["S"])
        np.testing.assert_array_equal(row["idx"], base[i]["idx"])
    prev = None
    for nb in range(1, 7):
        rows = oracle.block_index(wl, nb=nb)
        if prev is not None:
            for a, b in zip(prev, rows):
                assert set(a["cand"].tolist()) <= set(b["cand"].tolist())
                va, vb = a["val"][a["idx"] >= 0], b["val"][b["idx"] >= 0]
                assert len(vb) >= len(va)
                if len(va):
                    assert np.all(np.sort(vb)[::-1][:len(va)] >= np.sort(va)[::-1] - 1e-15)
        prev = rows
