"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
in test_oracle_pins.py catch every one of them."""
import numpy as np
import pytest

import oracle
import tests.test_oracle_pins as pins


def _pins_fail(monkeypatch, name, fn) -> bool:
    monkeypatch.setattr(oracle, name, fn)
    checks = [pins.test_golden_pooled_keys, pins.test_pool_ramp_and_partial_tail,
              pins.test_pool_two_sequences_offsets, pins.test_routing_every_head_is_dense_dsa,
              pins.test_hier_with_whole_prefix_is_dsa_topk,
              pins.test_topk_brute_force_with_ties_and_negative_zero,
              pins.test_single_block_router_is_dsa_of_mean_key, pins.test_selection_invariants]
    checks += [lambda c=c: pins.test_golden_case(c) for c in range(6)]
    checks += [lambda s=s: pins.test_brute_force_tiny(s) for s in range(3)]
    checks += [lambda c=c: pins.test_block_golden_case(c) for c in range(4)]
    checks += [lambda s=s: pins.test_block_brute_force_tiny(s) for s in range(4)]
    checks += [pins.test_block_pruning_keeping_every_block_is_routed_topk,
               pins.test_block_pruning_with_one_key_blocks_is_routed_topk]
    for chk in checks:
        try:
            chk()
        except AssertionError:
            return True
    return False


_orig_pool = oracle.pool_keys
_orig_router = oracle.router_scores
_orig_scores = oracle.token_scores
_orig_topk = oracle.topk
_orig_partial = oracle.partial_block_mean
_orig_block_scores = oracle.block_scores
_orig_block_query = oracle.block_pruned_query


def _pool_divide_by_B(K, key_offsets, B):
    out = _orig_pool(K, key_offsets, B).astype(np.float64)
    boff = oracle.block_offsets(key_offsets, B)
    for s in range(len(key_offsets) - 1):
        L = int(key_offsets[s + 1] - key_offsets[s])
        if L % B:
            out[boff[s + 1] - 1] *= (L % B) / B
    return out.astype(np.float32)


def _router_unsigned_w(q_t, w_t, K_seq, Kbar_seq, t, B):
    return _orig_router(q_t, np.abs(w_t), K_seq, Kbar_seq, t, B)


def _router_no_relu(q_t, w_t, K_seq, Kbar_seq, t, B):
    n = t + 1
    full = n // B
    aff = (q_t @ Kbar_seq[:full].astype(np.float64).T).sum(axis=1) if full else 0.0
    part = _orig_partial(K_seq, t, B)
    if part is not None:
        aff = aff + q_t @ part
    return w_t * aff


def _router_causal_leak(q_t, w_t, K_seq, Kbar_seq, t, B):
    # uses the whole block containing t (future keys) instead of the partial mean
    n = t + 1
    M = -(-n // B)
    dots = q_t @ Kbar_seq[:M].astype(np.float64).T
    return w_t * np.maximum(dots, 0.0).sum(axis=1)


def _partial_off_by_one(K_seq, t, B):
    n = t + 1
    full = n // B
    if n % B == 0:
        return None
    return K_seq[full * B:n + 1].mean(axis=0)


def _scores_no_relu(q_sel, w_sel, K_prefix):
    return w_sel @ (q_sel @ K_prefix.T)


def _scores_relu_after_weight(q_sel, w_sel, K_prefix):
    return np.maximum(w_sel[:, None] * (q_sel @ K_prefix.T), 0.0).sum(axis=0)


def _topk_ties_to_higher_index(I, k):
    n = I.shape[0]
    order = np.lexsort((-np.arange(n), -(I + 0.0)))[:k]
    idx = np.full(k, -1, dtype=np.int32)
    val = np.full(k, -np.inf)
    idx[:len(order)] = order
    val[:len(order)] = I[order]
    return idx, val


def _topk_ascending(I, k):
    idx, val = _orig_topk(-I, k)
    return idx, np.where(idx >= 0, -val, val)


def _block_scores_no_relu(q_sel, w_sel, Kbar_seq, t, B):
    full = (t + 1) // B
    return w_sel @ (q_sel @ Kbar_seq[:full].astype(np.float64).T)


def _block_scores_unsigned_w(q_sel, w_sel, Kbar_seq, t, B):
    return _orig_block_scores(q_sel, np.abs(w_sel), Kbar_seq, t, B)


def _block_scores_leak(q_sel, w_sel, Kbar_seq, t, B):
    # scores the pooled row of the query's own block too (it holds future keys)
    full = min(len(Kbar_seq), (t + B) // B)
    dots = q_sel @ Kbar_seq[:full].astype(np.float64).T
    return w_sel @ np.maximum(dots, 0.0)


def _block_query_drops_own_block(q_t, w_t, K_seq, Kbar_seq, t, B, m, nb, k, heads=None,
                                 blocks=None):
    res = _orig_block_query(q_t, w_t, K_seq, Kbar_seq, t, B, m, nb, k, heads, blocks)
    full = (t + 1) // B
    cand = res["cand"][res["cand"] < full * B]
    fine = oracle.hier_rerank_query(q_t[res["heads"]], w_t[res["heads"]], K_seq, cand, k)
    return res | dict(cand=cand, idx=fine["idx"], val=fine["val"])


def _block_query_keeps_worst(q_t, w_t, K_seq, Kbar_seq, t, B, m, nb, k, heads=None,
                             blocks=None):
    r = oracle.router_scores(q_t, w_t, K_seq, Kbar_seq, t, B)
    hs = oracle.route(r, m) if heads is None else heads
    S = oracle.block_scores(q_t[hs], w_t[hs], Kbar_seq, t, B)
    worst, _ = _orig_topk(-S, nb)
    return _orig_block_query(q_t, w_t, K_seq, Kbar_seq, t, B, m, nb, k, hs, worst)


MUTANTS = [
    ("pool_keys", _pool_divide_by_B),
    ("router_scores", _router_unsigned_w),
    ("router_scores", _router_no_relu),
    ("router_scores", _router_causal_leak),
    ("partial_block_mean", _partial_off_by_one),
    ("token_scores", _scores_no_relu),
    ("token_scores", _scores_relu_after_weight),
    ("topk", _topk_ties_to_higher_index),
    ("topk", _topk_ascending),
    ("block_scores", _block_scores_no_relu),
    ("block_scores", _block_scores_unsigned_w),
    ("block_scores", _block_scores_leak),
    ("block_pruned_query", _block_query_drops_own_block),
    ("block_pruned_query", _block_query_keeps_worst),
]


@pytest.mark.parametrize("name,fn", MUTANTS, ids=[f"{n}:{f.__name__}" for n, f in MUTANTS])
def test_pins_catch_planted_mistake(monkeypatch, name, fn):
    assert _pins_fail(monkeypatch, name, fn), f"no pin caught mutant {fn.__name__}"
