"""The tensor-core router (chosen for prefill-sized problems) vs the CPU
oracle on every row, through the C ABI (B200 only)."""
import numpy as np
import pytest
import torch

import long_context_sparse_misa_b200 as misa
from misa_synth import make_workload
from tests import parity

pytestmark = pytest.mark.gpu


def route_all(wl):
    prob = misa.Problem.from_workload(wl)
    K = torch.from_numpy(wl.K_bits).cuda()
    q = torch.from_numpy(wl.q_bits).cuda()
    w = torch.from_numpy(wl.w).cuda()
    ix = misa.Indexer(prob, m=wl.m, k=wl.k, with_router_scores=True)
    misa.profile_enable(True)
    ix.pool_route(q, w, K)
    prof = misa.profile_collect()
    misa.profile_enable(False)
    code, bits = misa.stream_status()
    assert code == 0, bits
    assert "route_split" in prof, "tensor-core router was not taken"
    return ix


def check(wl, ix):
    heads = ix.heads.cpu().numpy()
    rep = parity.check_misa_rows(wl, range(wl.T), np.zeros((wl.T, wl.k), np.int32),
                                 np.zeros((wl.T, wl.k), np.float32), heads=heads,
                                 r=ix.r.cpu().numpy(), Kbar=ix.Kbar.cpu().numpy())
    bad = [f for f in rep.failures if "router" in f or "head" in f or "Kbar" in f]
    assert not bad, bad
    q_r, w_r = ix.q_r.cpu().numpy(), ix.w_r.cpu().numpy()
    for i in range(0, wl.T, 97):
        np.testing.assert_array_equal(q_r[i], wl.q_bits[i][heads[i]])
        np.testing.assert_array_equal(w_r[i], wl.w[i][heads[i]])
    return rep


@pytest.mark.parametrize("H,B", [(64, 64), (32, 128), (16, 64), (8, 32)])
def test_route_tc_prefill(H, B):
    wl = make_workload(seq_lens=[3000], queries="all", H=H, B=B, m=8 if H >= 8 else H, k=64,
                       seed=H + B)
    rep = check(wl, route_all(wl))
    print(f"H={H}: head swaps {rep.head_swaps}, max router err / tol {rep.max_r_err:.3f}")


def test_route_tc_ragged_blocks_and_sequences():
    wl = make_workload(seq_lens=[1500, 1300, 5], queries="all", H=64, B=100, m=8, k=64, seed=3)
    check(wl, route_all(wl))


def test_route_tc_nonconsecutive_positions():
    L = 20000
    pos = np.arange(3, L, 7)
    wl = make_workload(seq_lens=[L], queries=[pos], H=32, B=128, m=8, k=64, seed=5)
    check(wl, route_all(wl))
