"""misa_route_static (router scratch in a library-owned device array) against
misa_route with a caller workspace, through the C ABI (B200 only).

The file name sorts last so that these calls also run after every other GPU
test in the same process; each test passes on its own as well.
"""
import numpy as np
import pytest
import torch

import long_context_sparse_misa_b200 as misa
from misa_synth import make_config, make_workload

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-4, 1e-3


def _inputs(wl):
    prob = misa.Problem.from_workload(wl)
    K = torch.from_numpy(wl.K_bits).cuda()
    q = torch.from_numpy(wl.q_bits).cuda()
    w = torch.from_numpy(wl.w).cuda()
    Kbar = torch.empty((prob.total_blocks, wl.d), dtype=torch.float32, device="cuda")
    misa.pool_keys(prob, K, Kbar)
    return prob, K, q, w, Kbar


def _outputs(wl, fill):
    T, H, m, d = wl.T, wl.H, wl.m, wl.d
    return (torch.full((T, m), fill, dtype=torch.int32, device="cuda"),
            torch.full((T, m, d), fill, dtype=torch.int16, device="cuda"),
            torch.full((T, m), float(fill), dtype=torch.float32, device="cuda"),
            torch.full((T, H), float(fill), dtype=torch.float32, device="cuda"))


def _status_ok():
    code, bits = misa.stream_status()
    assert code == 0 and bits == 0, f"device status {code}/{bits}"


def _compare_two_calls(wl):
    prob, K, q, w, Kbar = _inputs(wl)
    ws = torch.empty(misa.workspace_size(prob, wl.m, wl.k, 0), dtype=torch.uint8, device="cuda")
    ref = _outputs(wl, 0)
    misa.route(prob, q, w, K, Kbar, wl.m, *ref, ws)
    _status_ok()
    for call, fill in enumerate((-7, 3)):  # two calls in a row, different stale contents
        out = _outputs(wl, fill)
        misa.route_static(prob, q, w, K, Kbar, wl.m, *out)
        _status_ok()
        assert torch.equal(out[0], ref[0]), f"call {call}: routed heads differ"
        assert torch.equal(out[1], ref[1]), f"call {call}: q_r differs"
        torch.testing.assert_close(out[2], ref[2], atol=ATOL, rtol=RTOL)
        torch.testing.assert_close(out[3], ref[3], atol=ATOL, rtol=RTOL)


def test_static_router_decode_batch():
    # 16 sequences x 32K keys, 3 queries each: the CUDA-core router with
    # pooled-block ranges.
    _compare_two_calls(make_config(1))


def test_static_router_prefill_tensor_cores():
    # 6000 queries over one 6000-key prefix, H=32: the tcgen05 router, whose
    # scratch (group table, split pooled keys, a running block mean per key)
    # still fits the static array.
    wl = make_workload(seq_lens=[6000], queries="all", H=32, B=128, m=8, k=2048, seed=77)
    _compare_two_calls(wl)


def test_static_router_rejects_oversized_problem():
    # 300000 queries need a group table larger than the 4 MiB static scratch;
    # the call is refused on the host before any launch.
    T = 300000
    prob = misa.Problem([T], np.array([0, T], np.int32), np.arange(T, dtype=np.int32),
                        num_heads=8, block=128)
    dummy = torch.zeros(64, dtype=torch.float32, device="cuda")
    with pytest.raises(misa.MisaError) as e:
        misa.route_static(prob, dummy, dummy, dummy, dummy, 8, dummy, dummy, dummy, None)
    assert e.value.code == 2  # UNSUPPORTED
    assert "static scratch holds" in str(e.value)
