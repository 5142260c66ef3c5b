"""The agreement procedure of tests/parity.py on CPU: a correct selection
passes, and each planted mistake in a GPU-side row (a far swap, a duplicate,
bad padding, a wrong value, a token outside the candidates) is reported."""
import numpy as np

import oracle
from tests import parity


def _row(I, k, tokens=None):
    tokens = np.arange(len(I)) if tokens is None else np.asarray(tokens)
    idx, val = oracle.topk(np.asarray(I, np.float64), k)
    out = np.where(idx >= 0, tokens[np.maximum(idx, 0)], -1).astype(np.int32)
    return out, val.astype(np.float32)


def _check(I, idx, val, k, tokens=None):
    rep = parity.Report()
    parity.check_topk(rep, 0, np.asarray(I, np.float64), idx, val, k, tokens=tokens)
    return rep


def test_exact_selection_passes_in_any_row_order():
    rng = np.random.default_rng(0)
    I = rng.standard_normal(500)
    idx, val = _row(I, 40)
    perm = rng.permutation(40)
    rep = _check(I, idx[perm], val[perm], 40)
    assert not rep.failures and rep.topk_swaps == 0


def test_short_prefix_is_padded():
    I = np.array([0.5, -1.0, 2.0])
    idx, val = _row(I, 6)
    assert not _check(I, idx, val, 6).failures
    bad = val.copy()
    bad[-1] = 0.0
    assert "padding" in _check(I, idx, bad, 6).failures[0]


def test_far_swap_fails_and_near_tie_is_counted():
    I = np.linspace(0.0, 1.0, 200)
    idx, val = _row(I, 10)
    far = idx.copy()
    far[0] = 3  # a low score in place of a top one
    rep = _check(I, far, np.array([I[x] for x in far], np.float32), 10)
    assert rep.failures and "far from k-th" in rep.failures[0]
    J = I.copy()
    J[150] = J[idx[-1]] + 1e-6  # nearly tied with the k-th
    idx2, _ = _row(J, 10)
    swapped = idx2.copy()
    kth = int(np.argsort(-J, kind="stable")[9])
    other = 150 if kth != 150 else int(idx[-1])
    swapped[list(swapped).index(kth)] = other
    rep = _check(J, swapped, np.array([J[x] for x in swapped], np.float32), 10)
    assert not rep.failures and rep.topk_swaps == 1


def test_duplicate_wrong_value_and_foreign_token_fail():
    rng = np.random.default_rng(1)
    I = rng.standard_normal(300)
    idx, val = _row(I, 20)
    dup = idx.copy()
    dup[1] = dup[0]
    assert "distinct" in _check(I, dup, val, 20).failures[0]
    off = val.copy()
    off[5] += 0.01
    assert "value of token" in _check(I, idx, off, 20).failures[0]
    tokens = np.arange(0, 600, 2)  # candidates are the even tokens
    idx_t, val_t = _row(I, 20, tokens)
    assert not _check(I, idx_t, val_t, 20, tokens=tokens).failures
    odd = idx_t.copy()
    odd[0] += 1
    assert "outside" in _check(I, odd, val_t, 20, tokens=tokens).failures[0]
