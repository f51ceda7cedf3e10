"""Expert-parallel layer on one GPU (a one-rank NCCL group): every step in the library's kernels, the rows through
the NCCL all-to-all (collected after the single-GPU parity suites).  With one rank every expert is local, and each row's result does not depend on the rows
that share its tile, so the layer must reproduce moe_layer_decode bit for bit."""
import socket

import pytest
import torch
import torch.distributed as dist

from weight_only_bit_route_b200 import ep
from weight_only_bit_route_b200 import moe

from problems import build, dev_bf16, device_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def one_rank_group():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, init_method=f"tcp://127.0.0.1:{port}")
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("cfg", [1, 2])
def test_expert_parallel_one_rank_matches_layer(one_rank_group, cfg):
    P = build(cfg, "random")
    wl = P.wl
    L = device_layer(moe, P)
    ws = moe.workspace(P.T, wl.H, wl.E, wl.F, wl.k)
    x = dev_bf16(P.x)
    y_ref = moe.layer_decode(x, L, ws)
    layer = ep.ExpertParallelMoE(L.gate, L.up, L.down, L.router_w, top_k=wl.k, router_bias=L.router_bias,
                                 shared=L.shared, max_tokens=P.T)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert moe.read_status(ws) == 0
    assert torch.equal(y, y_ref)
    # ragged: fewer tokens through the same layer object
    y2 = layer.forward(x[:5].contiguous())
    y2_ref = moe.layer_decode(x[:5].contiguous(), L, moe.workspace(5, wl.H, wl.E, wl.F, wl.k))
    torch.cuda.synchronize()
    assert torch.equal(y2, y2_ref)
