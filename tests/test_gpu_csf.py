"""GPU parity of the compressed scale format (CSF) against the oracle.

"Step-5-Preview-NVFP4-Local", Format: the CSF planes (fixed, exceptions,
starts) encode the E4M3 block scales bit for bit; Size: the loader expands one
layer's scales into scratch when the layer runs.  Bars: bit-exact planes from
the encoder, bit-exact bytes from the decoder, and a layer run on decoded
scales bit-identical to the same layer on the raw scales.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_bit_route_b200 import moe
from weight_only_bit_route_b200 import synthetic as syn

from problems import build, dev, dev_bf16, device_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()


def _u32(t):
    return t.cpu().numpy().view(np.uint32)


CASES = ["random_E3_R32_C96", "random_E2_R16_C10_bytes_path", "constant_rows", "nvfp4_gate_E4", "nvfp4_down_E4"]


def _scales(name):
    rng = np.random.default_rng(11)
    if name == "random_E3_R32_C96":
        return rng.integers(0, 256, size=(3, 32, 96), dtype=np.uint8)
    if name == "random_E2_R16_C10_bytes_path":
        return rng.integers(0, 256, size=(2, 16, 10), dtype=np.uint8)
    if name == "constant_rows":
        return np.full((1, 16, 64), 250, np.uint8)
    # library-quantised NVFP4 scales at the pages' gate/up and down shapes (4 experts)
    which = name.split("_")[1]
    R, C = (1536, 256) if which == "gate" else (4096, 96)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    g = torch.Generator(device="cuda")
    mats = []
    for e in range(4):
        g.manual_seed(1000 + e)
        w = (torch.randn(R, C * 16, generator=g, device="cuda") * syn.WORKLOADS[1].w_std).to(torch.bfloat16)
        mats.append(moe.quantize_nvfp4(w, ws)[1])
    return torch.stack(mats).cpu().numpy()


@pytest.mark.parametrize("name", CASES)
def test_csf_encode_decode_bitexact(name):
    sc = _scales(name)
    E, R, C = sc.shape
    f_ref, e_ref, s_ref = oracle.csf_encode(sc)
    f, e, s = moe.csf_encode(dev(sc))
    torch.cuda.synchronize()
    assert np.array_equal(f.cpu().numpy(), f_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(_u32(e), e_ref)
    # decoder on the oracle's planes
    out = moe.csf_decode(dev(f_ref), dev(e_ref.view(np.int32)), dev(s_ref), R, C)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), sc)
    print(f"{name}: {len(e_ref)} exceptions in {sc.size} bytes")


def test_csf_decode_only_routed_experts():
    rng = np.random.default_rng(12)
    E, R, C = 6, 32, 96
    sc = rng.integers(0x20, 0x60, size=(E, R, C), dtype=np.uint8)
    f, e, s = oracle.csf_encode(sc)
    offsets = np.array([0, 3, 3, 9, 9, 9, 10], np.int32)          # experts 0, 2, 5 have rows
    out = torch.full((E, R, C), 0xAB, dtype=torch.uint8, device="cuda")
    moe.csf_decode(dev(f), dev(e.view(np.int32)), dev(s), R, C, expert_offsets=dev(offsets), out=out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    for ee in range(E):
        if offsets[ee + 1] > offsets[ee]:
            assert np.array_equal(got[ee], sc[ee])
        else:
            assert np.all(got[ee] == 0xAB)


def test_layer_on_csf_decoded_scales_is_identical():
    base = syn.WORKLOADS[0]
    wl = syn.Workload("tiny_nvfp4_T16", 16, base.H, base.E, base.F, base.k, "nvfp4", False, base.router_std, False)
    P = build(wl, "quantised", shared=True)
    L = device_layer(moe, P)
    ws = moe.workspace(P.T, wl.H, wl.E, wl.F, wl.k)
    x = dev_bf16(P.x)
    y_raw = moe.layer_decode(x, L, ws).clone()
    for bank in (L.gate, L.up, L.down):
        E, R, C = bank.scales.shape
        f, e, s = moe.csf_encode(bank.scales)
        bank.scales = moe.csf_decode(f, e, s, R, C)
    y_csf = moe.layer_decode(x, L, ws)
    torch.cuda.synchronize()
    assert moe.read_status(ws) == 0
    assert torch.equal(y_raw, y_csf)

