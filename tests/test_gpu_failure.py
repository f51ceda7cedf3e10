"""Failure handling on the GPU, without faulting it.

1. Bounded waits: with the workspace's hold set, the MMA warp of each
   tensor-core GEMM waits on a barrier nothing completes; with the wait bound
   at 1 ms that wait runs out.  The call must record MOE_ERR_TIMEOUT, the
   kernels must stop, drain the copies they have in flight and return (the
   context stays usable), and once the hold and the bound are cleared the same
   workspace must give the oracle's result.
2. A non-finite activation row on the 8-bit int4 path records
   MOE_ERR_NONFINITE and yields NaN for that token's rows only.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_bit_route_b200 import moe
from weight_only_bit_route_b200 import synthetic as syn

from problems import bf16_bits, build, dev, dev_bf16, device_bank, device_layer, layer_check, layer_tolerance

pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = -4
MOE_ERR_NONFINITE = -7


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()


def test_wait_limit_runs_out_then_recovers():
    P = build(0, "quantised", shared=True)
    wl = P.wl
    L = device_layer(moe, P)
    ws = moe.workspace(P.T, wl.H, wl.E, wl.F, wl.k)
    x = dev_bf16(P.x)
    moe.set_wait_limit(ws, 1_000_000)             # 1 ms
    moe.set_wait_hold(ws, 1)
    moe.layer_decode(x, L, ws)
    torch.cuda.synchronize()                       # the kernels returned
    assert moe.read_status(ws) == MOE_ERR_TIMEOUT
    moe.set_wait_hold(ws, 0)
    moe.set_wait_limit(ws, 0)
    for _ in range(2):                             # the workspace serves later calls
        y = moe.layer_decode(x, L, ws)
        ids, w = moe.route_topk(x, L.router_w, L.router_bias, wl.k, ws)
        torch.cuda.synchronize()
        assert moe.read_status(ws) == 0
        layer_check(P, bf16_bits(y), np.arange(P.T, dtype=np.int32), ids.cpu().numpy(), w.cpu().numpy())


def test_nonfinite_activation_row_is_reported():
    base = syn.WORKLOADS[0]
    wl = syn.Workload("tiny_int4_T16_inf", 16, base.H, base.E, base.F, base.k, "int4", False, base.router_std, False)
    P = build(wl, "quantised")
    off, rs, sr = oracle.permute(P.ids, wl.E)
    R = wl.T * wl.k
    bad = 5
    x = P.x.copy()
    x[bad, 17] = 0x7F80                             # +inf in bf16
    ref = oracle.grouped_swiglu(P.x, off, rs, wl.k, P.banks["gate"], P.banks["up"], np.arange(R))
    ws = moe.workspace(wl.T, wl.H, wl.E, wl.F, wl.k)
    g, u = device_bank(moe, P.banks["gate"]), device_bank(moe, P.banks["up"])
    h = moe.grouped_swiglu(dev_bf16(x), dev(off), dev(rs), wl.k, g, u, R, ws)   # 128 rows: the 8-bit path
    torch.cuda.synchronize()
    assert moe.read_status(ws) == MOE_ERR_NONFINITE
    got = oracle.bf16_to_f32(bf16_bits(h)).astype(np.float64)
    of_bad = (rs // wl.k) == bad
    assert np.all(np.isnan(got[of_bad]))
    assert np.all(np.abs(got[~of_bad] - ref[~of_bad]) <= layer_tolerance(ref[~of_bad]))
    # the same call without the infinity is clean
    h = moe.grouped_swiglu(dev_bf16(P.x), dev(off), dev(rs), wl.k, g, u, R, ws)
    torch.cuda.synchronize()
    assert moe.read_status(ws) == 0
