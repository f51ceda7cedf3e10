"""GPU parity of the NVFP4 W4A4 path against the oracle.

"Step-5-Preview-NVFP4-Local", Modifications: layers 3-87 are quant_algo NVFP4
(group size 16) with an input_scale, so the activations entering each routed
projection are NVFP4-quantised on the fly.  Bars: the activation quantiser is
bit-exact (codes and block scales); the per-step and layer outputs are within
|gpu - oracle| <= 1e-2 * max|oracle| + one bf16 ulp (the down step is fed the
GPU's own bf16 h, so both sides quantise the same values).
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_bit_route_b200 import moe
from weight_only_bit_route_b200 import synthetic as syn

from problems import bf16_bits, build, check_ids, dev, dev_bf16, device_bank, device_layer, layer_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()


def test_quantize_nvfp4_act_bitexact():
    rng = np.random.default_rng(3)
    x = syn.to_bf16_bits(rng.standard_normal((64, 1024)).astype(np.float32) * 2.0)
    g = (rng.uniform(0.2, 2.0, 64) * 4.0 / 2688).astype(np.float32)
    g[:4] = 1e-5                                        # saturating rows
    p_ref, s_ref, _ = oracle.act_quant_nvfp4(x, g)
    p, s = moe.quantize_nvfp4_act(dev_bf16(x), dev(g))
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(p.cpu().numpy(), p_ref)


def _in_scales(E, amax, seed):
    rng = np.random.default_rng(seed)
    return (amax / 2688.0 * rng.uniform(0.8, 1.25, E)).astype(np.float32)


def _tiny(T, E=None):
    base = syn.WORKLOADS[0]
    return syn.Workload(f"tiny_w4a4_T{T}", T, base.H, E or base.E, base.F, base.k, "nvfp4", False, base.router_std,
                        False)


@pytest.mark.parametrize("T", [16, 96])
def test_grouped_steps_w4a4(T):
    wl = _tiny(T)
    P = build(wl, "quantised")
    off, rs, sr = oracle.permute(P.ids, wl.E)
    R = wl.T * wl.k
    in_gu = _in_scales(wl.E, 4.0, 1)
    ref_h = oracle.grouped_swiglu_w4a4(P.x, off, rs, wl.k, P.banks["gate"], P.banks["up"], in_gu, np.arange(R))
    ws = moe.workspace(wl.T, wl.H, wl.E, wl.F, wl.k)
    g, u, d = (device_bank(moe, P.banks[w]) for w in ("gate", "up", "down"))
    g.input_scale = dev(in_gu)
    h = moe.grouped_swiglu(dev_bf16(P.x), dev(off), dev(rs), wl.k, g, u, R, ws)
    torch.cuda.synchronize()
    hb = bf16_bits(h)
    got = oracle.bf16_to_f32(hb).astype(np.float64)
    assert np.all(np.abs(got - ref_h) <= layer_tolerance(ref_h))
    # the W4A4 result is not the W4A16 one
    ref16 = oracle.grouped_swiglu(P.x, off, rs, wl.k, P.banks["gate"], P.banks["up"], np.arange(R))
    assert np.max(np.abs(ref_h - ref16)) > 1e-3 * np.max(np.abs(ref16))
    in_dn = _in_scales(wl.E, float(np.max(np.abs(got))), 2)
    d.input_scale = dev(in_dn)
    tw = P.w.ravel()
    ref_y = oracle.grouped_down_w4a4(hb, off, rs, tw, P.banks["down"], in_dn, np.arange(R))
    y = moe.grouped_down(h, dev(off), dev(rs), dev(tw), d, ws)
    torch.cuda.synchronize()
    assert moe.read_status(ws) == 0
    gy = oracle.bf16_to_f32(bf16_bits(y)).astype(np.float64)
    assert np.all(np.abs(gy - ref_y) <= layer_tolerance(ref_y))


def _w4a4_layer_check(P, L, in_gu, in_dn, tokens, T_all=None):
    wl = P.wl
    ws = moe.workspace(P.T, wl.H, wl.E, wl.F, wl.k)
    x = dev_bf16(P.x)
    y = moe.layer_forward(x, L, ws) if P.T > 64 else moe.layer_decode(x, L, ws)
    ids, w = moe.route_topk(x, L.router_w, L.router_bias, wl.k, ws)
    torch.cuda.synchronize()
    assert moe.read_status(ws) == 0
    ids_g, w_g = ids.cpu().numpy(), w.cpu().numpy()
    nt, _ = check_ids(ids_g[tokens], P, tokens)
    ids_o, w_o = P.ids.copy(), P.w.copy()
    for i in nt:
        ids_o[tokens[i]] = ids_g[tokens[i]]
        w_o[tokens[i]] = w_g[tokens[i]]
    ref = oracle.moe_forward_w4a4(P.x, ids_o, w_o, P.banks["gate"], P.banks["up"], P.banks["down"], in_gu, in_dn,
                                  shared=P.shared, tokens=tokens)
    got = oracle.bf16_to_f32(bf16_bits(y)[tokens]).astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= layer_tolerance(ref)), f"max err {err.max()} vs {1e-2 * np.max(np.abs(ref))}"
    return float(err.max() / np.max(np.abs(ref)))


@pytest.mark.parametrize("T", [16, 100])
def test_layer_w4a4_all_tokens(T):
    wl = _tiny(T)
    P = build(wl, "quantised", shared=True)
    L = device_layer(moe, P)
    in_gu, in_dn = _in_scales(wl.E, 4.0, 3), _in_scales(wl.E, 1.0, 4)
    L.gate.input_scale = dev(in_gu)
    L.down.input_scale = dev(in_dn)
    rel = _w4a4_layer_check(P, L, in_gu, in_dn, np.arange(P.T, dtype=np.int32))
    print(f"T={T}: max rel err {rel:.2e}")


def test_layer_w4a4_full_size_decode():
    """The decode workload's shapes (T = 8, H = 4096, E = 352, F = 1536, BF16 shared
    expert) with W4A4 routed experts: all 8 tokens."""
    P = build(2, "random")
    wl = P.wl
    L = device_layer(moe, P)
    in_gu, in_dn = _in_scales(wl.E, 4.5, 5), _in_scales(wl.E, 2.0, 6)
    L.gate.input_scale = dev(in_gu)
    L.down.input_scale = dev(in_dn)
    rel = _w4a4_layer_check(P, L, in_gu, in_dn, np.arange(P.T, dtype=np.int32))
    print(f"decode W4A4: max rel err {rel:.2e}")


def test_w4a4_rejects_other_formats_and_split_scales():
    P = build(0, "quantised")
    L = device_layer(moe, P)                             # int4 banks
    ws = moe.workspace(P.T, P.wl.H, P.wl.E, P.wl.F, P.wl.k)
    L.gate.input_scale = torch.ones(P.wl.E, device="cuda")
    with pytest.raises(moe.MoEError):
        moe.layer_decode(dev_bf16(P.x), L, ws)
