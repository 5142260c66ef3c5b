"""Python binding of libmisa, the B200 (sm_100a) MISA routed sparse-attention indexer.

Argument marshalling only: every step of the indexer runs in the CUDA
kernels behind the C ABI declared in include/misa.h.  PyTorch provides
device memory and streams.  There is no CPU fallback: importing this package
without a built libmisa.so raises ImportError (build it with
``python long_context_sparse_misa_b200/build.py``).

Method: "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
Inference" -- a block-pooled router keeps m of the H indexer heads per query,
only those heads score the causal prefix, and a per-query top-k follows;
MISA-dagger re-ranks an enlarged candidate set with all H heads; block
pruning lets the routed heads score only the tokens of the best pooled
blocks.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "LIB_PATH", "lib", "MisaError", "Problem", "workspace_size", "block_offsets", "pool_keys",
    "route", "pool_keys_from", "score_topk", "hier_rerank", "dsa_index_dense", "stream_status",
    "selftest_timeout", "route_static", "EXPORTED", "Indexer", "profile_enable", "profile_collect",
    "block_workspace_size", "block_score_topk",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmisa.so")

# Every symbol include/misa.h declares.
EXPORTED = (
    "misa_workspace_size", "misa_block_offsets", "misa_pool_keys", "misa_pool_keys_from",
    "misa_route",
    "misa_route_static", "misa_score_topk", "misa_hier_rerank", "dsa_index_dense", "misa_stream_status",
    "misa_selftest_timeout", "misa_profile_enable", "misa_profile_collect",
    "misa_last_error_string", "misa_block_workspace_size", "misa_block_score_topk",
)

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python long_context_sparse_misa_b200/build.py` (needs nvcc)")
lib = ctypes.CDLL(LIB_PATH)

_c_i32, _c_i64, _c_sz, _c_p = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p


class _Problem(ctypes.Structure):
    _fields_ = [
        ("num_seqs", _c_i32), ("num_queries", _c_i32), ("num_heads", _c_i32),
        ("head_dim", _c_i32), ("block", _c_i32), ("max_seq_len", _c_i32),
        ("total_keys", _c_i64), ("total_blocks", _c_i64),
        ("key_offsets", _c_p), ("block_offsets", _c_p), ("query_offsets", _c_p),
        ("q_pos", _c_p),
    ]


_PP = ctypes.POINTER(_Problem)
_sig = {
    "misa_workspace_size": (_c_sz, [_PP, _c_i32, _c_i32, _c_i32]),
    "misa_block_offsets": (ctypes.c_int, [_c_p, _c_i32, _c_i32, _c_p, _c_p]),
    "misa_pool_keys": (ctypes.c_int, [_PP, _c_p, _c_p, _c_p]),
    "misa_pool_keys_from": (ctypes.c_int, [_PP, _c_p, _c_p, _c_p, _c_p]),
    "misa_route": (ctypes.c_int, [_PP, _c_p, _c_p, _c_p, _c_p, _c_i32, _c_p, _c_p, _c_p, _c_p,
                                  _c_p, _c_sz, _c_p]),
    "misa_route_static": (ctypes.c_int, [_PP, _c_p, _c_p, _c_p, _c_p, _c_i32, _c_p, _c_p, _c_p,
                                         _c_p, _c_p]),
    "misa_score_topk": (ctypes.c_int, [_PP, _c_p, _c_p, _c_i32, _c_p, _c_i32, _c_p, _c_p, _c_p,
                                       _c_i64, _c_p, _c_sz, _c_p]),
    "misa_hier_rerank": (ctypes.c_int, [_PP, _c_p, _c_p, _c_p, _c_p, _c_i32, _c_i32, _c_p, _c_p,
                                        _c_p, _c_sz, _c_p]),
    "dsa_index_dense": (ctypes.c_int, [_PP, _c_p, _c_p, _c_p, _c_i32, _c_p, _c_p, _c_p, _c_i64,
                                       _c_p, _c_sz, _c_p]),
    "misa_stream_status": (ctypes.c_int, [_c_p, ctypes.POINTER(_c_i32)]),
    "misa_selftest_timeout": (ctypes.c_int, [_c_i32, _c_p]),
    "misa_profile_enable": (ctypes.c_int, [_c_i32]),
    "misa_profile_collect": (ctypes.c_int, [_c_i32, ctypes.c_char_p, ctypes.POINTER(ctypes.c_double),
                                            ctypes.POINTER(_c_i64)]),
    "misa_last_error_string": (ctypes.c_char_p, []),
    "misa_block_workspace_size": (_c_sz, [_PP, _c_i32]),
    "misa_block_score_topk": (ctypes.c_int, [_PP, _c_p, _c_p, _c_i32, _c_p, _c_p, _c_i32, _c_i32,
                                             _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(lib, _name)
    _f.restype, _f.argtypes = _res, _args

ERR_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "WORKSPACE_TOO_SMALL", 4: "CUDA",
             5: "DEVICE_TIMEOUT", 6: "DEVICE_BOUNDS", 7: "DEVICE_BAD_INPUT"}


class MisaError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = lib.misa_last_error_string().decode(errors="replace")
        super().__init__(f"{where}: {ERR_NAMES.get(code, code)}: {msg}")
        self.code = code


def _check(code: int, where: str) -> None:
    if code != 0:
        raise MisaError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Problem:
    """Shapes of one indexer call plus its device metadata.

    Built from host metadata: per-sequence key counts, per-sequence query
    counts and the query positions.  The offsets are uploaded to the device
    and block offsets are computed there by misa_block_offsets.
    """

    def __init__(self, seq_lens, query_offsets, q_pos, num_heads: int, block: int,
                 device="cuda", head_dim: int = 128, stream=None):
        import numpy as np
        import torch
        seq_lens = np.asarray(seq_lens, dtype=np.int64)
        ko = np.zeros(len(seq_lens) + 1, dtype=np.int64)
        ko[1:] = np.cumsum(seq_lens)
        self.seq_lens = seq_lens
        self.key_offsets = torch.from_numpy(ko).to(device)
        self.query_offsets = torch.from_numpy(np.asarray(query_offsets, np.int32)).to(device)
        self.q_pos = torch.from_numpy(np.asarray(q_pos, np.int32)).to(device)
        self.block_offsets = torch.empty(len(seq_lens) + 1, dtype=torch.int64, device=device)
        nblocks = int(np.sum((seq_lens + block - 1) // block))
        self.c = _Problem(
            num_seqs=len(seq_lens), num_queries=len(q_pos), num_heads=num_heads,
            head_dim=head_dim, block=block, max_seq_len=int(max(1, seq_lens.max(initial=1))),
            total_keys=int(ko[-1]), total_blocks=nblocks,
            key_offsets=self.key_offsets.data_ptr(), block_offsets=self.block_offsets.data_ptr(),
            query_offsets=self.query_offsets.data_ptr(),
            q_pos=self.q_pos.data_ptr() if len(q_pos) else None)
        block_offsets(self.key_offsets, len(seq_lens), block, self.block_offsets, stream)

    @classmethod
    def from_workload(cls, wl, device="cuda", stream=None):
        return cls(wl.seq_lens, wl.query_offsets, wl.q_pos, wl.H, wl.B, device=device,
                   head_dim=wl.d, stream=stream)

    @property
    def ref(self):
        return ctypes.byref(self.c)

    @property
    def T(self):
        return self.c.num_queries

    @property
    def H(self):
        return self.c.num_heads

    @property
    def total_blocks(self):
        return self.c.total_blocks


def workspace_size(prob: Problem, m: int, k: int, k_cand: int = 0) -> int:
    n = lib.misa_workspace_size(prob.ref, m, k, k_cand)
    if n == 0:
        raise MisaError(1, "misa_workspace_size")
    return int(n)


def block_offsets(key_offsets, num_seqs: int, block: int, out, stream=None) -> None:
    _check(lib.misa_block_offsets(_ptr(key_offsets), num_seqs, block, _ptr(out), _stream(stream)),
           "misa_block_offsets")


def pool_keys(prob: Problem, K, Kbar, stream=None) -> None:
    _check(lib.misa_pool_keys(prob.ref, _ptr(K), _ptr(Kbar), _stream(stream)), "misa_pool_keys")


def pool_keys_from(prob: Problem, K, Kbar, from_pos, stream=None) -> None:
    _check(lib.misa_pool_keys_from(prob.ref, _ptr(K), _ptr(Kbar), _ptr(from_pos),
                                   _stream(stream)), "misa_pool_keys_from")


def route(prob: Problem, q, w, K, Kbar, m: int, heads, q_r, w_r, router_scores, ws,
          stream=None) -> None:
    _check(lib.misa_route(prob.ref, _ptr(q), _ptr(w), _ptr(K), _ptr(Kbar), m, _ptr(heads),
                          _ptr(q_r), _ptr(w_r), _ptr(router_scores), _ptr(ws), ws.numel(),
                          _stream(stream)), "misa_route")


def route_static(prob: Problem, q, w, K, Kbar, m: int, heads, q_r, w_r, router_scores,
                 stream=None) -> None:
    _check(lib.misa_route_static(prob.ref, _ptr(q), _ptr(w), _ptr(K), _ptr(Kbar), m,
                                 _ptr(heads), _ptr(q_r), _ptr(w_r), _ptr(router_scores),
                                 _stream(stream)), "misa_route_static")


def score_topk(prob: Problem, q_r, w_r, m: int, K, k: int, idx, val, ws, scores_dbg=None,
               stream=None) -> None:
    ld = 0 if scores_dbg is None else scores_dbg.stride(0)
    _check(lib.misa_score_topk(prob.ref, _ptr(q_r), _ptr(w_r), m, _ptr(K), k, _ptr(idx),
                               _ptr(val), _ptr(scores_dbg), ld, _ptr(ws), ws.numel(),
                               _stream(stream)), "misa_score_topk")


def hier_rerank(prob: Problem, q, w, K, cand, k_cand: int, k: int, idx, val, ws,
                stream=None) -> None:
    _check(lib.misa_hier_rerank(prob.ref, _ptr(q), _ptr(w), _ptr(K), _ptr(cand), k_cand, k,
                                _ptr(idx), _ptr(val), _ptr(ws), ws.numel(), _stream(stream)),
           "misa_hier_rerank")


def dsa_index_dense(prob: Problem, q, w, K, k: int, idx, val, ws, scores_dbg=None,
                    stream=None) -> None:
    ld = 0 if scores_dbg is None else scores_dbg.stride(0)
    _check(lib.dsa_index_dense(prob.ref, _ptr(q), _ptr(w), _ptr(K), k, _ptr(idx), _ptr(val),
                               _ptr(scores_dbg), ld, _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_index_dense")


def block_workspace_size(prob: Problem, n_blocks: int) -> int:
    n = lib.misa_block_workspace_size(prob.ref, n_blocks)
    if n == 0:
        raise MisaError(1, "misa_block_workspace_size")
    return int(n)


def block_score_topk(prob: Problem, q_r, w_r, m: int, K, Kbar, n_blocks: int, k: int, idx, val,
                     ws, blocks=None, stream=None) -> None:
    _check(lib.misa_block_score_topk(prob.ref, _ptr(q_r), _ptr(w_r), m, _ptr(K), _ptr(Kbar),
                                     n_blocks, k, _ptr(idx), _ptr(val), _ptr(blocks), _ptr(ws),
                                     ws.numel(), _stream(stream)), "misa_block_score_topk")


def stream_status(stream=None) -> int:
    """Synchronise the stream; return (code, status bits) and clear the status word."""
    st = _c_i32(0)
    code = lib.misa_stream_status(_stream(stream), ctypes.byref(st))
    return code, st.value


def profile_enable(on: bool = True) -> None:
    """Bracket every library kernel launch of this thread with CUDA events."""
    lib.misa_profile_enable(1 if on else 0)


def profile_collect(max_kernels: int = 64) -> dict:
    """Synchronise and return {kernel name: (total ms, launches)}; clears the record."""
    names = ctypes.create_string_buffer(32 * max_kernels)
    ms = (ctypes.c_double * max_kernels)()
    cnt = (_c_i64 * max_kernels)()
    n = lib.misa_profile_collect(max_kernels, names, ms, cnt)
    if n < 0:
        raise MisaError(-n, "misa_profile_collect")
    out = {}
    for i in range(n):
        nm = names.raw[32 * i:32 * i + 32].split(b"\0", 1)[0].decode()
        out[nm] = (float(ms[i]), int(cnt[i]))
    return out


def selftest_timeout(wait_ms: int, stream=None) -> None:
    _check(lib.misa_selftest_timeout(wait_ms, _stream(stream)), "misa_selftest_timeout")


class Indexer:
    """Owns the device buffers of one problem and runs the call sequences.

    misa():   pool_keys -> route -> score_topk            (MISA)
    hier():   pool_keys -> route -> score_topk(k_cand) -> hier_rerank (MISA-dagger)
    dense():  dsa_index_dense                             (the DSA indexer)
    blocks(): pool_keys -> route -> block_score_topk      (routed heads x block pruning;
              needs n_blocks at construction)
    All inputs are device tensors: K uint16/bf16 [total_keys, 128],
    q [T, H, 128] bf16 bits, w [T, H] float32.
    """

    def __init__(self, prob: Problem, m: int, k: int, k_cand: int = 0, device="cuda",
                 with_router_scores: bool = False, n_blocks: int = 0):
        import torch
        self.prob, self.m, self.k, self.k_cand = prob, m, k, k_cand
        T, H = prob.T, prob.H
        dev = device
        self.ws = torch.empty(workspace_size(prob, m, max(k, k_cand), k_cand), dtype=torch.uint8,
                              device=dev)
        self.Kbar = torch.empty((max(prob.total_blocks, 1), 128), dtype=torch.float32, device=dev)
        self.heads = torch.empty((T, m), dtype=torch.int32, device=dev)
        self.q_r = torch.empty((T, m, 128), dtype=torch.uint16, device=dev)
        self.w_r = torch.empty((T, m), dtype=torch.float32, device=dev)
        self.r = (torch.empty((T, H), dtype=torch.float32, device=dev)
                  if with_router_scores else None)
        self.idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        self.val = torch.empty((T, k), dtype=torch.float32, device=dev)
        if k_cand:
            self.cand = torch.empty((T, k_cand), dtype=torch.int32, device=dev)
            self.cand_val = torch.empty((T, k_cand), dtype=torch.float32, device=dev)
        self.n_blocks = n_blocks
        if n_blocks:
            self.block_ws = torch.empty(block_workspace_size(prob, n_blocks), dtype=torch.uint8,
                                        device=dev)
            self.blocks_kept = torch.empty((T, n_blocks), dtype=torch.int32, device=dev)

    def pool_route(self, q, w, K, stream=None, pool_from=None):
        """pool_from: None re-pools every block; else an int32 device tensor
        [S] of first new key positions (Kbar must hold the earlier blocks)."""
        if pool_from is None:
            pool_keys(self.prob, K, self.Kbar, stream)
        else:
            pool_keys_from(self.prob, K, self.Kbar, pool_from, stream)
        route(self.prob, q, w, K, self.Kbar, self.m, self.heads, self.q_r, self.w_r, self.r,
              self.ws, stream)

    def misa(self, q, w, K, stream=None, scores_dbg=None, pool_from=None):
        self.pool_route(q, w, K, stream, pool_from)
        score_topk(self.prob, self.q_r, self.w_r, self.m, K, self.k, self.idx, self.val,
                   self.ws, scores_dbg, stream)
        return self.idx, self.val

    def hier(self, q, w, K, stream=None, pool_from=None):
        self.pool_route(q, w, K, stream, pool_from)
        score_topk(self.prob, self.q_r, self.w_r, self.m, K, self.k_cand, self.cand,
                   self.cand_val, self.ws, None, stream)
        hier_rerank(self.prob, q, w, K, self.cand, self.k_cand, self.k, self.idx, self.val,
                    self.ws, stream)
        return self.idx, self.val

    def blocks(self, q, w, K, stream=None, pool_from=None):
        self.pool_route(q, w, K, stream, pool_from)
        block_score_topk(self.prob, self.q_r, self.w_r, self.m, K, self.Kbar, self.n_blocks,
                         self.k, self.idx, self.val, self.block_ws, self.blocks_kept, stream)
        return self.idx, self.val

    def dense(self, q, w, K, stream=None, scores_dbg=None):
        dsa_index_dense(self.prob, q, w, K, self.k, self.idx, self.val, self.ws, scores_dbg,
                        stream)
        return self.idx, self.val
