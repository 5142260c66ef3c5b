"""Seeded synthetic workloads for the MISA routed indexer.

This module is the one piece shared by the CPU oracle and the CUDA path. It
only draws random numbers and lays them out; it holds none of the method's
arithmetic (no pooling, routing, scoring or selection).

Value recipe (stand-in for DeepSeek-V3.2 / GLM-5 indexer activations, whose
weights and prompts are not available):
  * q[t, h, :] and k[s, :] ~ N(0, 1) / sqrt(d) elementwise, drawn in fp32 and
    rounded to bf16 with round-to-nearest-even.
  * w[t, h] ~ N(0, 1) / sqrt(H), kept in fp32.
  * "Needles": per sequence, P = round(0.01 * L) positions drawn without
    replacement; each picks one head h_s uniform in [0, H) and gets
    k[s] += 2 * u_{h_s} in fp32 before the bf16 rounding, where u_h is a
    seeded random unit vector (normalised N(0, I_d)).
  * Streams: numpy PCG64 seeded by SeedSequence([seed, i]) with
    i = 0 keys, 1 queries, 2 head weights, 3 needle directions,
    4 needle positions, 5 needle heads.  seed = 1000 + config index.

Layout handed to both sides (host numpy arrays):
  K_bits      uint16 [sum_s L_s, d]   bf16 bit patterns, sequences packed
  q_bits      uint16 [T, H, d]        bf16 bit patterns
  w           float32 [T, H]
  key_offsets int64  [S + 1]          rows of K owned by sequence s
  query_offsets int32 [S + 1]         queries of sequence s
  q_pos       int32  [T]              position t of each query; it sees keys 0..t
"""
from __future__ import annotations

import dataclasses
import math
from typing import Sequence

import numpy as np

__all__ = [
    "CONFIGS", "Workload", "make_config", "make_workload",
    "f32_to_bf16_bits", "bf16_bits_to_f32",
]

# The five workloads of the routed-indexer study: decode (tiny and batched),
# prefill at 32K and 128K, and hierarchical decode at 128K.
CONFIGS = [
    dict(name="tiny_decode_L4096_q64_H64", S=1, L=4096, queries=64, H=64, d=128,
         B=64, m=8, k=256, k_cand=0),
    dict(name="decode_batch_16x32K_q3_H64", S=16, L=32768, queries=3, H=64, d=128,
         B=64, m=8, k=2048, k_cand=0),
    dict(name="prefill_32K_H64", S=1, L=32768, queries="all", H=64, d=128,
         B=64, m=8, k=2048, k_cand=0),
    dict(name="prefill_128K_H32", S=1, L=131072, queries="all", H=32, d=128,
         B=128, m=8, k=2048, k_cand=0),
    dict(name="hier_decode_8x128K_H64", S=8, L=131072, queries=1, H=64, d=128,
         B=128, m=8, k=2048, k_cand=8192),
]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    out = ((u + rounding) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 exactly."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Workload:
    name: str
    K_bits: np.ndarray
    q_bits: np.ndarray
    w: np.ndarray
    key_offsets: np.ndarray
    query_offsets: np.ndarray
    q_pos: np.ndarray
    H: int
    d: int
    B: int
    m: int
    k: int
    k_cand: int = 0

    @property
    def S(self) -> int:
        return len(self.key_offsets) - 1

    @property
    def T(self) -> int:
        return len(self.q_pos)

    @property
    def seq_lens(self) -> np.ndarray:
        return np.diff(self.key_offsets)

    @property
    def q_seq(self) -> np.ndarray:
        """Sequence id of every query (expanded from query_offsets)."""
        return np.repeat(np.arange(self.S, dtype=np.int32), np.diff(self.query_offsets))

    @property
    def pairs(self) -> int:
        """Scored (query, prefix-token) pairs: sum over queries of t + 1."""
        return int(np.sum(self.q_pos.astype(np.int64) + 1))

    def subset_queries(self, rows: Sequence[int]) -> "Workload":
        """Same keys, only the listed query rows (rows must be sorted)."""
        rows = np.asarray(rows, dtype=np.int64)
        seq = self.q_seq[rows]
        qo = np.zeros(self.S + 1, dtype=np.int32)
        np.add.at(qo, seq + 1, 1)
        qo = np.cumsum(qo).astype(np.int32)
        return dataclasses.replace(
            self, q_bits=self.q_bits[rows], w=self.w[rows], q_pos=self.q_pos[rows],
            query_offsets=qo)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))


def make_workload(*, seq_lens: Sequence[int], queries, H: int, d: int = 128, B: int = 64,
                  m: int = 8, k: int = 2048, k_cand: int = 0, seed: int = 0,
                  needles: bool = True, name: str = "custom") -> Workload:
    """Draw one seeded workload.

    queries: "all" (every position of every sequence), an int Q (the last Q
    positions of each sequence), or a list with one position list per sequence.
    """
    seq_lens = [int(x) for x in seq_lens]
    S = len(seq_lens)
    key_offsets = np.zeros(S + 1, dtype=np.int64)
    key_offsets[1:] = np.cumsum(seq_lens)
    total = int(key_offsets[-1])

    if isinstance(queries, str):
        if queries != "all":
            raise ValueError(queries)
        pos = [np.arange(L, dtype=np.int32) for L in seq_lens]
    elif isinstance(queries, (int, np.integer)):
        pos = [np.arange(max(L - int(queries), 0), L, dtype=np.int32) for L in seq_lens]
    else:
        pos = [np.asarray(p, dtype=np.int32) for p in queries]
        if len(pos) != S:
            raise ValueError("one position list per sequence")
    query_offsets = np.zeros(S + 1, dtype=np.int32)
    query_offsets[1:] = np.cumsum([len(p) for p in pos])
    q_pos = np.concatenate(pos) if pos else np.zeros(0, np.int32)
    T = len(q_pos)

    K = _rng(seed, 0).standard_normal((total, d), dtype=np.float32)
    K *= np.float32(1.0 / math.sqrt(d))
    if needles:
        u = _rng(seed, 3).standard_normal((H, d), dtype=np.float32)
        u /= np.linalg.norm(u, axis=1, keepdims=True).astype(np.float32)
        r_pos, r_head = _rng(seed, 4), _rng(seed, 5)
        for s, L in enumerate(seq_lens):
            P = int(round(0.01 * L))
            if P == 0:
                continue
            where = r_pos.choice(L, size=P, replace=False)
            heads = r_head.integers(0, H, size=P)
            K[key_offsets[s] + where] += np.float32(2.0) * u[heads]
    K_bits = f32_to_bf16_bits(K)
    del K

    q = _rng(seed, 1).standard_normal((T, H, d), dtype=np.float32)
    q *= np.float32(1.0 / math.sqrt(d))
    q_bits = f32_to_bf16_bits(q)
    del q
    w = _rng(seed, 2).standard_normal((T, H), dtype=np.float32)
    w *= np.float32(1.0 / math.sqrt(H))

    return Workload(name=name, K_bits=K_bits, q_bits=q_bits, w=w, key_offsets=key_offsets,
                    query_offsets=query_offsets, q_pos=q_pos.astype(np.int32), H=H, d=d, B=B,
                    m=m, k=k, k_cand=k_cand)


def make_config(index: int, seed: int | None = None) -> Workload:
    """The full-size workload of one of the five configurations."""
    c = CONFIGS[index]
    return make_workload(seq_lens=[c["L"]] * c["S"], queries=c["queries"], H=c["H"], d=c["d"],
                         B=c["B"], m=c["m"], k=c["k"], k_cand=c["k_cand"],
                         seed=1000 + index if seed is None else seed, name=c["name"])
