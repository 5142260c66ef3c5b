"""CPU oracle for the MISA routed sparse-attention indexer.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
cpu_baseline / reference leg of bench.py may import this package.  The CUDA
library never calls it, and it shares no code, table or helper with the CUDA
path; the only thing both sides use is the seeded input generator in
misa_synth (random numbers and layout, no arithmetic of the method).

What it computes, in the order the method runs, from
"MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference":
  1. pool_keys      mean-pooled key blocks           (gist.science summary,
                    "Methodologie: MISA", Lightweight Block-Pooled Router)
  2. router_scores  per-head importance from pooled keys, then route() keeps
                    the top-m heads                  (same passage)
  3. token_scores   routed token-level scoring       (same section,
                    Sparse Token Scoring; abstract)
  4. topk           per-query top-k                  (same passage)
  5. hier_rerank    MISA-dagger coarse-to-fine re-rank with all heads
                    (gist.science summary, "Hierarchische Variant (MISA†)")
  6. dense_index    the dense all-head DSA indexer    (abstract; summary,
                    "Probleemstelling")
  7. recall_iou     token recovery vs DSA, measured as IoU
                    (summary, "Experimentele Resultaten", Token Recovery)
  8. block_pruned_query  head axis x token axis: after routing, the routed
                    heads score the pooled blocks, only the best blocks'
                    tokens are scored (thelatestinai.com papers page, HISA
                    abstract: block-level coarse filter on pooled blocks,
                    then the indexer inside the kept blocks; gist.science
                    summary, "Probleemstelling" and "Betekenis en Claims":
                    head-axis routing combines with token-axis schemes)

Precision: inputs are the same bytes the GPU sees (bf16 bit patterns widened
exactly, fp32 head weights widened exactly); every dot product, sum and mean
is evaluated in fp64.  Pooled keys are rounded once to fp32, which is their
contract value.  Selection is a full sort by (score descending, index
ascending) -- the plain definition, no selection trick.

Readings the pages leave open (each restated where it is used):
  * The DSA indexer score is I[t,s] = sum_h w[t,h] * ReLU(q[t,h] . k[s]).  The
    pages name the token-wise indexer and its heads but print no formula;
    this is DeepSeek-V3.2's lightning-indexer score.
  * Router aggregation: r[t,h] = w[t,h] * sum_b ReLU(q[t,h] . Kbar_t[b]) over
    the blocks query t can see (the head's own indexer term evaluated on
    pooled keys, summed, unweighted, with the signed head weight).  The
    method is training-free, so the router has no learned parameters.
  * Causality: query t sees keys 0..t (self included).  It uses the
    floor((t+1)/B) full blocks from the pooled table plus, when (t+1) is not
    a multiple of B, one partial block averaged over its visible keys only.
  * Ties: heads by (r desc, head asc); tokens by (I desc, index asc);
    -0 counts as +0.  A prefix shorter than k selects every token and pads
    with index -1 / value -inf.
  * Block pruning (8.): the block score is the routed heads' indexer score
    of the pooled key, over the full blocks the query sees; the nb best
    blocks by (score desc, block asc) are kept, and the query's own
    incomplete block (keys floor((t+1)/B)*B .. t), when there is one, is
    always kept.

Parity status: every function here is pinned by tests/test_oracle_pins.py
(closed forms, hand-worked examples, brute force on tiny inputs, identities
the pages state).  The whole pipeline against the pages' own numbers is
parity unpinned: the pages print no worked example, and their 92% / 3.82x
figures come from trained models and another GPU.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "widen_bf16", "pool_keys", "block_offsets", "partial_block_mean", "router_scores",
    "route", "token_scores", "topk", "misa_query", "misa_index", "dense_query",
    "dense_index", "hier_rerank_query", "hier_index", "recall_iou", "block_scores",
    "block_pruned_query", "block_index",
]


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact fp64 values."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def block_offsets(key_offsets: np.ndarray, B: int) -> np.ndarray:
    """Row offset of each sequence's first pooled block: M_s = ceil(L_s / B)
    blocks per sequence (gist.science summary, "Methodologie: MISA":
    the prefix is split into M = ceil(L/B) blocks)."""
    L = np.diff(np.asarray(key_offsets, dtype=np.int64))
    M = (L + B - 1) // B
    out = np.zeros(len(L) + 1, dtype=np.int64)
    out[1:] = np.cumsum(M)
    return out


def pool_keys(K: np.ndarray, key_offsets: np.ndarray, B: int) -> np.ndarray:
    """Mean-pooled indexer keys, one row per block of B consecutive keys.

    Follows gist.science summary, "Methodologie: MISA" (Lightweight
    Block-Pooled Router: block-level statistics are mean-pooled indexer
    keys).  The last block of a sequence may hold fewer than B keys; it is
    the mean of the keys present.  Sums and the division are fp64; the
    result is rounded once to fp32.

    K: fp64 [sum L, d] (exact widened bf16).  Returns fp32 [sum ceil(L/B), d].
    """
    key_offsets = np.asarray(key_offsets, dtype=np.int64)
    boff = block_offsets(key_offsets, B)
    d = K.shape[1]
    out = np.zeros((int(boff[-1]), d), dtype=np.float32)
    for s in range(len(key_offsets) - 1):
        k0, k1 = int(key_offsets[s]), int(key_offsets[s + 1])
        for b in range(int(boff[s + 1] - boff[s])):
            lo = k0 + b * B
            hi = min(lo + B, k1)
            block = K[lo:hi]
            out[boff[s] + b] = (block.sum(axis=0) / float(hi - lo)).astype(np.float32)
    return out


def partial_block_mean(K_seq: np.ndarray, t: int, B: int) -> np.ndarray | None:
    """Causal partial block of query t: the mean of keys floor((t+1)/B)*B .. t,
    or None when t+1 is a multiple of B (no partial block).  fp64."""
    n = t + 1
    full = n // B
    if n % B == 0:
        return None
    return K_seq[full * B:n].sum(axis=0) / float(n - full * B)


def router_scores(q_t: np.ndarray, w_t: np.ndarray, K_seq: np.ndarray, Kbar_seq: np.ndarray,
                  t: int, B: int) -> np.ndarray:
    """Per-head importance of every indexer head for query t.

    gist.science summary, "Methodologie: MISA": per-head affinities are
    computed against the pooled block keys and aggregated into one
    importance score per head.  Reading adopted:
        r[h] = w[h] * sum_{b < M_t} ReLU(q[h] . Kbar_t[b])
    with M_t = ceil((t+1)/B); the full blocks come from the pooled table
    (its fp32 values), the partial block is the causal mean of the keys the
    query can see.

    q_t: fp64 [H, d]; w_t: fp64 [H]; K_seq: fp64 [L, d]; Kbar_seq: fp32 [M, d].
    Returns fp64 [H].
    """
    n = t + 1
    full = n // B
    aff = np.zeros(q_t.shape[0], dtype=np.float64)
    if full > 0:
        dots = q_t @ Kbar_seq[:full].astype(np.float64).T        # [H, full]
        aff += np.maximum(dots, 0.0).sum(axis=1)
    part = partial_block_mean(K_seq, t, B)
    if part is not None:
        aff += np.maximum(q_t @ part, 0.0)
    return w_t * aff


def route(r: np.ndarray, m: int) -> np.ndarray:
    """Keep the top-m heads by router score (gist.science summary,
    "Methodologie: MISA": the router selects the top-h heads).  Ties go to
    the lower head index.  Returns the head ids in rank order."""
    H = r.shape[0]
    order = np.lexsort((np.arange(H), -r))
    return order[:m].astype(np.int32)


def token_scores(q_sel: np.ndarray, w_sel: np.ndarray, K_prefix: np.ndarray) -> np.ndarray:
    """Token-level indexer scores with a set of heads.

    I[s] = sum_j w_sel[j] * ReLU(q_sel[j] . k[s]) for every key of the
    prefix.  With the routed heads this is MISA's sparse token scoring
    (gist.science summary, "Methodologie: MISA", Sparse Token Scoring);
    with all H heads it is the dense DSA indexer (abstract).

    q_sel: fp64 [h, d]; w_sel: fp64 [h]; K_prefix: fp64 [n, d] -> fp64 [n].
    """
    dots = q_sel @ K_prefix.T                                    # [h, n]
    return w_sel @ np.maximum(dots, 0.0)


def topk(I: np.ndarray, k: int) -> tuple[np.ndarray, np.ndarray]:
    """The min(k, n) largest scores by (score desc, index asc); -0 == +0.
    Rows shorter than k are padded with index -1 and value -inf.
    Returns (idx int32 [k], val float64 [k]) in rank order."""
    n = I.shape[0]
    I = I + 0.0                      # -0 -> +0
    order = np.lexsort((np.arange(n), -I))[:k]
    idx = np.full(k, -1, dtype=np.int32)
    val = np.full(k, -np.inf, dtype=np.float64)
    idx[:len(order)] = order
    val[:len(order)] = I[order]
    return idx, val


def _seq_arrays(wl, Kf: np.ndarray, Kbar: np.ndarray, s: int):
    k0, k1 = int(wl.key_offsets[s]), int(wl.key_offsets[s + 1])
    boff = block_offsets(wl.key_offsets, wl.B)
    return Kf[k0:k1], Kbar[boff[s]:boff[s + 1]]


def misa_query(q_t, w_t, K_seq, Kbar_seq, t, B, m, k, heads=None):
    """One query through MISA: route, score the prefix with the routed heads,
    select top-k.  `heads` overrides the router's choice (used by the parity
    harness to re-score with another implementation's head set).
    Returns dict(r, heads, I, idx, val)."""
    r = router_scores(q_t, w_t, K_seq, Kbar_seq, t, B)
    if heads is None:
        heads = route(r, m)
    I = token_scores(q_t[heads], w_t[heads], K_seq[:t + 1])
    idx, val = topk(I, k)
    return dict(r=r, heads=np.asarray(heads, dtype=np.int32), I=I, idx=idx, val=val)


def dense_query(q_t, w_t, K_seq, t, k):
    """One query through the dense DSA indexer: all heads, top-k."""
    I = token_scores(q_t, w_t, K_seq[:t + 1])
    idx, val = topk(I, k)
    return dict(I=I, idx=idx, val=val)


def hier_rerank_query(q_t, w_t, K_seq, cand, k):
    """MISA-dagger fine stage (gist.science summary, "Hierarchische Variant
    (MISA†)"): the original all-head DSA indexer re-scores only the candidate
    tokens and keeps the final top-k.  Candidates with index -1 are padding.
    Ties go to the lower token index.  Returns dict(I_cand, idx, val)."""
    cand = np.asarray(cand, dtype=np.int64)
    cand = np.sort(cand[cand >= 0])
    I_c = token_scores(q_t, w_t, K_seq[cand]) + 0.0
    order = np.lexsort((cand, -I_c))[:k]
    idx = np.full(k, -1, dtype=np.int32)
    val = np.full(k, -np.inf, dtype=np.float64)
    idx[:len(order)] = cand[order]
    val[:len(order)] = I_c[order]
    return dict(I_cand=I_c, idx=idx, val=val)


def _rows(wl, rows):
    return range(wl.T) if rows is None else rows


def misa_index(wl, rows=None, m=None, k=None):
    """MISA over the listed query rows of a misa_synth.Workload.
    Returns dict(Kbar, per-row results)."""
    m = wl.m if m is None else m
    k = wl.k if k is None else k
    Kf = widen_bf16(wl.K_bits)
    Kbar = pool_keys(Kf, wl.key_offsets, wl.B)
    qs = wl.q_seq
    out = []
    for i in _rows(wl, rows):
        s = int(qs[i])
        K_seq, Kbar_seq = _seq_arrays(wl, Kf, Kbar, s)
        out.append(misa_query(widen_bf16(wl.q_bits[i]), wl.w[i].astype(np.float64), K_seq,
                              Kbar_seq, int(wl.q_pos[i]), wl.B, m, k))
    return dict(Kbar=Kbar, rows=out)


def dense_index(wl, rows=None, k=None):
    """Dense DSA indexer over the listed query rows."""
    k = wl.k if k is None else k
    Kf = widen_bf16(wl.K_bits)
    qs = wl.q_seq
    out = []
    for i in _rows(wl, rows):
        s = int(qs[i])
        K_seq = Kf[int(wl.key_offsets[s]):int(wl.key_offsets[s + 1])]
        out.append(dense_query(widen_bf16(wl.q_bits[i]), wl.w[i].astype(np.float64), K_seq,
                               int(wl.q_pos[i]), k))
    return out


def hier_index(wl, rows=None, m=None, k_cand=None, k=None):
    """MISA-dagger: the routed pass keeps k_cand candidates, all heads re-rank
    them to the final top-k."""
    m = wl.m if m is None else m
    k_cand = wl.k_cand if k_cand is None else k_cand
    k = wl.k if k is None else k
    coarse = misa_index(wl, rows, m=m, k=k_cand)
    Kf = widen_bf16(wl.K_bits)
    qs = wl.q_seq
    out = []
    for j, i in enumerate(_rows(wl, rows)):
        s = int(qs[i])
        K_seq = Kf[int(wl.key_offsets[s]):int(wl.key_offsets[s + 1])]
        fine = hier_rerank_query(widen_bf16(wl.q_bits[i]), wl.w[i].astype(np.float64), K_seq,
                                 coarse["rows"][j]["idx"], k)
        fine["coarse"] = coarse["rows"][j]
        out.append(fine)
    return out


def recall_iou(A, D) -> tuple[float, float]:
    """Token recovery of selection A against the DSA selection D: recall
    |A n D| / |D| and IoU |A n D| / |A u D| (gist.science summary,
    "Experimentele Resultaten", Token Recovery, measured by IoU).
    Index -1 is padding and is ignored.  Empty D gives (1, 1)."""
    a = set(int(x) for x in np.asarray(A).ravel() if x >= 0)
    d = set(int(x) for x in np.asarray(D).ravel() if x >= 0)
    if not d and not a:
        return 1.0, 1.0
    inter = len(a & d)
    recall = inter / len(d) if d else 1.0
    return recall, inter / len(a | d)


def block_scores(q_sel: np.ndarray, w_sel: np.ndarray, Kbar_seq: np.ndarray, t: int,
                 B: int) -> np.ndarray:
    """Coarse stage of block pruning: the indexer score of every full pooled
    block query t can see, with a set of heads,
        S[b] = sum_j w_sel[j] * ReLU(q_sel[j] . Kbar[b]),  b < floor((t+1)/B)
    (thelatestinai.com papers page, HISA abstract: pooled block
    representations are scored to drop irrelevant regions).  The full
    blocks' values are the pooled table's fp32 rows.

    q_sel: fp64 [h, d]; w_sel: fp64 [h]; Kbar_seq: fp32 [M, d] -> fp64 [full].
    """
    full = (t + 1) // B
    dots = q_sel @ Kbar_seq[:full].astype(np.float64).T          # [h, full]
    return w_sel @ np.maximum(dots, 0.0)


def block_pruned_query(q_t, w_t, K_seq, Kbar_seq, t, B, m, nb, k, heads=None, blocks=None):
    """One query through routed heads x block pruning.

    1. route (as misa_query), keep m heads;
    2. block_scores with the routed heads, keep the nb best full blocks by
       (score desc, block asc) -- `blocks` overrides that choice (the parity
       harness re-scores with another implementation's block set);
    3. candidates = the tokens of the kept blocks plus the query's own
       incomplete block (keys floor((t+1)/B)*B .. t);
    4. the routed heads score the candidates, top-k by (score desc, token
       asc) (thelatestinai.com papers page, HISA abstract: token-level
       refinement inside the kept blocks).
    Returns dict(r, heads, S, blocks, cand, idx, val).
    """
    r = router_scores(q_t, w_t, K_seq, Kbar_seq, t, B)
    if heads is None:
        heads = route(r, m)
    heads = np.asarray(heads, dtype=np.int64)
    S = block_scores(q_t[heads], w_t[heads], Kbar_seq, t, B)
    if blocks is None:
        blocks, _ = topk(S, nb)
    blocks = np.asarray(blocks, dtype=np.int64)
    full = (t + 1) // B
    kept = [int(b) for b in blocks if b >= 0]
    cand = [b * B + j for b in kept for j in range(B)]
    cand += list(range(full * B, t + 1))
    cand = np.array(sorted(cand), dtype=np.int64)
    fine = hier_rerank_query(q_t[heads], w_t[heads], K_seq, cand, k)
    return dict(r=r, heads=heads.astype(np.int32), S=S, blocks=blocks.astype(np.int32),
                cand=cand, idx=fine["idx"], val=fine["val"])


def block_index(wl, nb, rows=None, m=None, k=None):
    """Routed heads x block pruning over the listed query rows of a
    misa_synth.Workload, nb kept full blocks per query."""
    m = wl.m if m is None else m
    k = wl.k if k is None else k
    Kf = widen_bf16(wl.K_bits)
    Kbar = pool_keys(Kf, wl.key_offsets, wl.B)
    out = []
    for i in _rows(wl, rows):
        s = int(wl.q_seq[i])
        K_seq, Kbar_seq = _seq_arrays(wl, Kf, Kbar, s)
        out.append(block_pruned_query(widen_bf16(wl.q_bits[i]), wl.w[i].astype(np.float64),
                                      K_seq, Kbar_seq, int(wl.q_pos[i]), wl.B, m, nb, k))
    return out
