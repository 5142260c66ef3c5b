"""Agreement procedure between the CUDA indexer and the CPU oracle.

Floating point: |gpu - oracle| <= ATOL + RTOL * |oracle| with ATOL = 1e-4,
RTOL = 1e-3 (fp32 scores from bf16 inputs).  Integer results (routed head
sets, top-k index sets) must match exactly, except entries whose oracle
score lies within that tolerance of the m-th (heads) or k-th (tokens)
threshold; those swaps are counted and reported.  Where the router swapped
near-tied heads, the oracle re-scores the row with the GPU's head set, so a
single near-tie does not spoil the whole row.  Invariants checked on every
row: indices causal and distinct, exactly min(k, n) of them, every selected
score >= every unselected score (up to the tolerance).
"""
from __future__ import annotations

import dataclasses

import numpy as np

import oracle

ATOL, RTOL = 1e-4, 1e-3


def tol(x):
    return ATOL + RTOL * np.abs(x)


@dataclasses.dataclass
class Report:
    rows: int = 0
    head_swaps: int = 0
    topk_swaps: int = 0
    max_val_err: float = 0.0
    max_r_err: float = 0.0
    failures: list = dataclasses.field(default_factory=list)

    def fail(self, msg):
        if len(self.failures) < 20:
            self.failures.append(msg)

    def assert_ok(self):
        assert not self.failures, "\n".join(self.failures)


def check_heads(rep: Report, i, r_oracle, heads_gpu, m):
    """Set compare of routed heads; returns True when the GPU set is acceptable."""
    ref = oracle.route(r_oracle, m)
    g = set(int(h) for h in heads_gpu)
    o = set(int(h) for h in ref)
    if len(g) != m or any(h < 0 or h >= len(r_oracle) for h in g):
        rep.fail(f"row {i}: invalid head set {sorted(g)}")
        return False
    if g == o:
        return True
    thr = r_oracle[ref[-1]]
    for h in g ^ o:
        if abs(r_oracle[h] - thr) > tol(thr):
            rep.fail(f"row {i}: head {h} r={r_oracle[h]:.6g} far from m-th {thr:.6g}")
            return False
    rep.head_swaps += 1
    return True


def check_topk(rep: Report, i, I_oracle, idx_gpu, val_gpu, k, tokens=None):
    """Check one row of (idx, val) against oracle scores over `tokens`
    (sorted, distinct; default: the prefix 0..n-1 with I_oracle indexed by
    token)."""
    I_oracle = np.asarray(I_oracle, dtype=np.float64)
    n = len(I_oracle)
    tokens = np.arange(n) if tokens is None else np.asarray(tokens, dtype=np.int64)
    idx_gpu = np.asarray(idx_gpu)
    val_gpu = np.asarray(val_gpu)
    k_eff = min(k, n)
    valid = idx_gpu >= 0
    sel = idx_gpu[valid].astype(np.int64)
    if len(sel) != k_eff or len(np.unique(sel)) != k_eff:
        rep.fail(f"row {i}: {len(sel)} selected ({len(np.unique(sel))} distinct), expected {k_eff}")
        return
    where = np.searchsorted(tokens, sel)
    inside = (where < n) & (tokens[np.minimum(where, n - 1)] == sel)
    if not inside.all():
        rep.fail(f"row {i}: selected token outside the candidate/prefix set")
        return
    pad = np.flatnonzero(~valid)
    if len(pad) != k - k_eff or not np.all(np.isneginf(val_gpu[pad])):
        rep.fail(f"row {i}: bad padding")
    # values
    sv = I_oracle[where]
    gv = val_gpu[valid].astype(np.float64)
    err = np.abs(gv - sv)
    if len(err):
        rep.max_val_err = max(rep.max_val_err, float((err / tol(sv)).max()))
        if np.any(err > tol(sv)):
            j = int(np.argmax(err - tol(sv)))
            rep.fail(f"row {i}: value of token {sel[j]} gpu={gv[j]:.7g} oracle={sv[j]:.7g}")
    # set compare with near-threshold allowance
    order = np.lexsort((tokens, -(I_oracle + 0.0)))[:k_eff]
    ref = set(tokens[order].tolist())
    g = set(sel.tolist())
    if g != ref and k_eff < n:
        thr = I_oracle[order[-1]]
        for x in g ^ ref:
            sx = I_oracle[int(np.searchsorted(tokens, x))]
            if abs(sx - thr) > tol(thr):
                rep.fail(f"row {i}: token {x} I={sx:.7g} far from k-th {thr:.7g}")
                return
        rep.topk_swaps += len(g - ref)
    # invariant: selected >= unselected (up to tolerance)
    if k_eff < n:
        unsel = np.ones(n, dtype=bool)
        unsel[where] = False
        umax = I_oracle[unsel].max()
        if sv.min() < umax - tol(umax):
            rep.fail(f"row {i}: selected min {sv.min():.7g} < unselected max {umax:.7g}")


def check_misa_rows(wl, rows, idx, val, heads=None, r=None, Kbar=None, k=None, m=None,
                    rep: Report | None = None):
    """MISA rows: router (if heads/r given), then top-k re-scored with the GPU's heads."""
    rep = rep or Report()
    k = wl.k if k is None else k
    m = wl.m if m is None else m
    Kf = oracle.widen_bf16(wl.K_bits)
    Kbar_o = oracle.pool_keys(Kf, wl.key_offsets, wl.B)
    if Kbar is not None:
        err = np.abs(Kbar - Kbar_o)
        if np.any(err > tol(Kbar_o)):
            rep.fail(f"Kbar mismatch, max err {err.max():.3g}")
    boff = oracle.block_offsets(wl.key_offsets, wl.B)
    qs = wl.q_seq
    for j, i in enumerate(rows):
        s = int(qs[i])
        t = int(wl.q_pos[i])
        K_seq = Kf[int(wl.key_offsets[s]):int(wl.key_offsets[s + 1])]
        q_t = oracle.widen_bf16(wl.q_bits[i])
        w_t = wl.w[i].astype(np.float64)
        r_o = oracle.router_scores(q_t, w_t, K_seq, Kbar_o[boff[s]:boff[s + 1]], t, wl.B)
        use = None
        if r is not None:
            e = np.abs(r[j] - r_o)
            rep.max_r_err = max(rep.max_r_err, float((e / tol(r_o)).max()))
            if np.any(e > tol(r_o)):
                rep.fail(f"row {i}: router score err {e.max():.3g}")
        if heads is not None:
            if not check_heads(rep, i, r_o, heads[j], m):
                continue
            use = np.asarray(heads[j], dtype=np.int64)
        else:
            use = oracle.route(r_o, m)
        I = oracle.token_scores(q_t[use], w_t[use], K_seq[:t + 1])
        check_topk(rep, i, I, idx[j], val[j], k)
        rep.rows += 1
    return rep


def check_dense_rows(wl, rows, idx, val, k=None, rep: Report | None = None):
    rep = rep or Report()
    k = wl.k if k is None else k
    Kf = oracle.widen_bf16(wl.K_bits)
    qs = wl.q_seq
    for j, i in enumerate(rows):
        s = int(qs[i])
        t = int(wl.q_pos[i])
        K_seq = Kf[int(wl.key_offsets[s]):int(wl.key_offsets[s + 1])]
        I = oracle.token_scores(oracle.widen_bf16(wl.q_bits[i]), wl.w[i].astype(np.float64),
                                K_seq[:t + 1])
        check_topk(rep, i, I, idx[j], val[j], k)
        rep.rows += 1
    return rep


def check_rerank_rows(wl, rows, cand, idx, val, k=None, rep: Report | None = None):
    """Re-rank of the GPU's own candidate rows against the oracle re-rank."""
    rep = rep or Report()
    k = wl.k if k is None else k
    Kf = oracle.widen_bf16(wl.K_bits)
    qs = wl.q_seq
    for j, i in enumerate(rows):
        s = int(qs[i])
        K_seq = Kf[int(wl.key_offsets[s]):int(wl.key_offsets[s + 1])]
        c = np.asarray(cand[j])
        c = np.sort(c[c >= 0])
        I_c = oracle.token_scores(oracle.widen_bf16(wl.q_bits[i]), wl.w[i].astype(np.float64),
                                  K_seq[c])
        check_topk(rep, i, I_c, idx[j], val[j], k, tokens=c)
        rep.rows += 1
    return rep


def check_block_set(rep: Report, i, S_oracle, blocks_gpu, nb):
    """Kept pooled blocks (routed heads x block pruning): a set compare with the
    same near-threshold allowance as the token top-k.  Returns True when the
    GPU's set is acceptable."""
    full = len(S_oracle)
    want = min(nb, full)
    g = [int(b) for b in blocks_gpu if b >= 0]
    if len(g) != want or len(set(g)) != want or any(b >= full for b in g):
        rep.fail(f"row {i}: kept blocks {sorted(g)} invalid ({want} of {full} expected)")
        return False
    if sum(1 for b in blocks_gpu if b < 0) != nb - want:
        rep.fail(f"row {i}: bad block padding")
        return False
    ref, _ = oracle.topk(np.asarray(S_oracle, dtype=np.float64), nb)
    o = set(int(b) for b in ref if b >= 0)
    if set(g) != o:
        thr = S_oracle[int(ref[want - 1])]
        for b in set(g) ^ o:
            if abs(S_oracle[b] - thr) > tol(thr):
                rep.fail(f"row {i}: block {b} S={S_oracle[b]:.7g} far from nb-th {thr:.7g}")
                return False
        rep.topk_swaps += len(set(g) - o)
    return True


def check_block_rows(wl, rows, heads, blocks, idx, val, nb, k=None, m=None,
                     rep: Report | None = None):
    """Routed heads x block pruning: heads against the oracle router, kept
    blocks against the oracle's block scores with the GPU's heads, then the
    top-k against the oracle's scores of the candidates the GPU's blocks give."""
    rep = rep or Report()
    k = wl.k if k is None else k
    m = wl.m if m is None else m
    Kf = oracle.widen_bf16(wl.K_bits)
    Kbar_o = oracle.pool_keys(Kf, wl.key_offsets, wl.B)
    boff = oracle.block_offsets(wl.key_offsets, wl.B)
    for j, i in enumerate(rows):
        s = int(wl.q_seq[i])
        t = int(wl.q_pos[i])
        K_seq = Kf[int(wl.key_offsets[s]):int(wl.key_offsets[s + 1])]
        Kbar_seq = Kbar_o[boff[s]:boff[s + 1]]
        q_t = oracle.widen_bf16(wl.q_bits[i])
        w_t = wl.w[i].astype(np.float64)
        r_o = oracle.router_scores(q_t, w_t, K_seq, Kbar_seq, t, wl.B)
        if not check_heads(rep, i, r_o, heads[j], m):
            continue
        use = np.asarray(heads[j], dtype=np.int64)
        S_o = oracle.block_scores(q_t[use], w_t[use], Kbar_seq, t, wl.B)
        if not check_block_set(rep, i, S_o, blocks[j], nb):
            continue
        res = oracle.block_pruned_query(q_t, w_t, K_seq, Kbar_seq, t, wl.B, m, nb, k,
                                        heads=use, blocks=blocks[j])
        c = res["cand"]
        I_c = oracle.token_scores(q_t[use], w_t[use], K_seq[c])
        check_topk(rep, i, I_c, idx[j], val[j], k, tokens=c)
        rep.rows += 1
    return rep
