"""The C-ABI library loads and exports every declared symbol; host-side
argument checks answer without a GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def misa():
    # The build script is loaded by path: importing the package needs the library.
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_misa_build", os.path.join(ROOT, "long_context_sparse_misa_b200", "build.py"))
    builder = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(builder)
    builder.build()
    import long_context_sparse_misa_b200 as m
    return m


def declared_functions():
    with open(os.path.join(ROOT, "include", "misa.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\*?\s+\*?(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points(misa):
    names = declared_functions()
    assert set(names) == set(misa.EXPORTED), names


def test_library_exports_every_declared_symbol(misa):
    lib = ctypes.CDLL(misa.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def _problem(misa, **kw):
    d = dict(num_seqs=1, num_queries=4, num_heads=64, head_dim=128, block=64, max_seq_len=1000,
             total_keys=1000, total_blocks=16, key_offsets=8, block_offsets=8, query_offsets=8,
             q_pos=8)
    d.update(kw)
    return misa._Problem(**d)


def test_workspace_size_and_validation(misa):
    p = _problem(misa)
    n = misa.lib.misa_workspace_size(ctypes.byref(p), 8, 2048, 0)
    assert n >= 4 * 1000 * 4
    assert misa.lib.misa_workspace_size(ctypes.byref(p), 65, 2048, 0) == 0      # m > H
    bad = _problem(misa, head_dim=64)
    assert misa.lib.misa_workspace_size(ctypes.byref(bad), 8, 10, 0) == 0
    assert b"head_dim" in misa.lib.misa_last_error_string()
    hier = misa.lib.misa_workspace_size(ctypes.byref(p), 8, 2048, 8192)
    assert hier >= 4 * 8192 * 4


def test_host_argument_errors_without_gpu(misa):
    p = _problem(misa)
    rp = ctypes.byref(p)
    lib = misa.lib
    # NULL pointers are rejected before any CUDA call
    assert lib.misa_route(rp, None, None, None, None, 8, None, None, None, None, None, 0, None) == 1
    assert lib.misa_score_topk(rp, None, None, 8, None, 16, None, None, None, 0, None, 0, None) == 1
    # m not a power of two -> UNSUPPORTED; k out of range -> INVALID_ARG
    assert lib.misa_score_topk(rp, 16, 16, 6, 16, 16, 16, 16, None, 0, 16, 1 << 20, None) == 2
    assert lib.misa_score_topk(rp, 16, 16, 8, 16, 0, 16, 16, None, 0, 16, 1 << 20, None) == 1
    # misaligned bf16 pointer
    assert lib.misa_score_topk(rp, 18, 16, 8, 16, 16, 16, 16, None, 0, 16, 1 << 20, None) == 1
    assert b"aligned" in lib.misa_last_error_string()
    # hierarchical: k_cand < k
    assert lib.misa_hier_rerank(rp, 16, 16, 16, 16, 10, 20, 16, 16, 16, 1 << 20, None) == 1
    # dense needs H a power of two
    p48 = _problem(misa, num_heads=48)
    assert lib.dsa_index_dense(ctypes.byref(p48), 16, 16, 16, 8, 16, 16, None, 0, 16, 1 << 20,
                               None) == 2
    # workspace too small
    assert lib.misa_route(rp, 16, 16, 16, 16, 8, 16, 16, 16, None, 16, 8, None) == 3
    assert lib.misa_selftest_timeout(0, None) == 1
    assert lib.misa_block_offsets(None, 1, 64, None, None) == 1
    # incremental pooling: NULL / misaligned arguments are rejected on the host
    assert lib.misa_pool_keys_from(rp, 16, 16, None, None) == 1
    assert b"from_pos" in lib.misa_last_error_string()
    assert lib.misa_pool_keys_from(rp, 16, 16, 18, None) == 1
    assert lib.misa_pool_keys_from(rp, 16, None, 16, None) == 1
    # the static-scratch router validates like misa_route and refuses m > H
    assert lib.misa_route_static(rp, 16, 16, 16, 16, 65, 16, 16, 16, None, None) == 1


def test_workspace_size_covers_the_selection_after_the_scoring_pass(misa):
    # 128K prefill, m = 8, k = 2048: candidate lists per query row (62 rows of
    # 128 lanes x 8 B) for the exact selection after the pass, plus the
    # double-buffered per-CTA lists and the rest (well under 4 GB more).
    T = 131072
    p = _problem(misa, num_queries=T, num_heads=32, block=128, max_seq_len=T, total_keys=T,
                 total_blocks=T // 128)
    n = misa.lib.misa_workspace_size(ctypes.byref(p), 8, 2048, 0)
    lists = T * 62 * 128 * 8
    assert lists <= n < lists + (4 << 30)
    # a larger k needs longer lists
    assert misa.lib.misa_workspace_size(ctypes.byref(p), 8, 8192, 0) > n
    # a decode batch does not stream: no per-query lists
    d = _problem(misa, num_seqs=16, num_queries=48, max_seq_len=32768, total_keys=16 * 32768,
                 total_blocks=16 * 512)
    assert misa.lib.misa_workspace_size(ctypes.byref(d), 8, 2048, 0) < 64 << 20


def test_block_pruning_arguments_and_workspace_without_gpu(misa):
    lib = misa.lib
    # decode batch 16 x 32K, B = 64, 64 kept blocks: score rows of 512 pooled
    # blocks, 65 x 64 candidates per query
    d = _problem(misa, num_seqs=16, num_queries=48, max_seq_len=32768, total_keys=16 * 32768,
                 total_blocks=16 * 512)
    rp = ctypes.byref(d)
    n = lib.misa_block_workspace_size(rp, 64)
    per_query = 2 * 512 * 4 + 2 * 64 * 4 + 2 * 65 * 64 * 4
    assert 48 * per_query <= n < 48 * per_query + 6 * 256
    assert lib.misa_block_workspace_size(rp, 0) == 0                 # n_blocks >= 1
    assert lib.misa_block_workspace_size(rp, 1024) == 0              # (n+1)*B > 65536
    assert b"n_blocks" in lib.misa_last_error_string()
    args = lambda m, nb, k, ws_bytes, q=16: lib.misa_block_score_topk(
        rp, q, 16, m, 16, 16, nb, k, 16, 16, None, 256, ws_bytes, None)
    assert args(6, 64, 2048, n) == 2           # m not a power of two
    assert args(128, 64, 2048, n) == 2         # m > H
    assert args(8, 64, 0, n) == 1              # k < 1
    assert args(8, 8, 2048, n) == 1            # k > (n_blocks + 1) * B
    assert args(8, 64, 2048, n, q=18) == 1     # misaligned q_r
    assert args(8, 64, 2048, n - 1) == 3       # workspace too small
