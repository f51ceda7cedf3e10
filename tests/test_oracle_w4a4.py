"""Pins for the oracle's NVFP4 W4A4 path ("Step-5-Preview-NVFP4-Local",
Modifications: layers 3-87 are quant_algo NVFP4, group size 16, with an
input_scale; layers 88-90 have none and keep BF16 activations).

The activation quantiser is the weight quantiser's block step with a given
global scale; it is pinned against the weight quantiser itself (a row whose
global is its own amax / (6 * 448)), against brute-force nearest codes with
torch's E4M3 conversion for the block scale (saturating at 448), and through
the special case where every activation is exactly representable (W4A4 then
equals W4A16).  The layer is pinned against a brute-force dense mixture over
all experts with per-expert activation quantisation.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_bit_route_b200 import synthetic as syn

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _bf16(a):
    return syn.to_bf16_bits(np.asarray(a, np.float32))


def test_act_quant_equals_weight_quantiser_on_its_own_global():
    rng = np.random.default_rng(0)
    for cols in (16, 256, 1024):
        row = _bf16(rng.standard_normal((1, cols)) * 0.7)
        p_w, s_w, g = oracle.quant_nvfp4(row)
        p_a, s_a, xq = oracle.act_quant_nvfp4(row, g)
        assert np.array_equal(p_a, p_w) and np.array_equal(s_a, s_w)
        assert np.array_equal(xq, oracle.dequant_nvfp4(p_w, s_w, g))


@pytest.mark.parametrize("g", [1e-3, 2.5e-4, 3e-6])
def test_act_quant_brute_force_nearest(g):
    """Block scale: E4M3 round-to-nearest-even of amax / (6 g), saturating at 448
    (torch float8_e4m3fn after clamping); each value: the nearest E2M1 multiple
    of the block scale (ties to the even code), saturating at 6."""
    rng = np.random.default_rng(1)
    x = _bf16(rng.standard_normal((8, 256)) * np.float32(1.0))
    packed, scales, xq = oracle.act_quant_nvfp4(x, g)
    xf = oracle.bf16_to_f32(x).astype(np.float32)
    gf = np.float32(g)
    for r in range(x.shape[0]):
        for b in range(x.shape[1] // 16):
            blk = xf[r, 16 * b:16 * b + 16]
            t = np.float32(np.max(np.abs(blk))) / (np.float32(6.0) * gf)
            sb = torch.tensor(min(float(t), 448.0)).to(torch.float8_e4m3fn).view(torch.uint8).item()
            assert scales[r, b] == sb, (r, b)
            eff = np.float32(torch.tensor(sb, dtype=torch.uint8).view(torch.float8_e4m3fn).float().item()) * gf
            for j in range(16):
                v = blk[j] / eff if eff > 0 else 0.0
                a = min(abs(float(v)), 6.0)
                d = np.abs(E2M1 - a)
                best = np.flatnonzero(d == d.min())
                code = best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]
                want = np.sign(v) * E2M1[code] if v != 0 else 0.0
                got_code = (packed[r, (16 * b + j) // 2] >> (4 * (j % 2))) & 0xF
                got = (-1 if got_code & 8 else 1) * E2M1[got_code & 7]
                assert got == want, (r, b, j, v, got, want)


def test_w4a4_equals_w4a16_when_activations_are_representable():
    """x built from E2M1 values times an exact block scale times g (each block
    holding a 6 so its scale is exactly reproduced): quantisation is the
    identity, so the W4A4 gate/up step equals the W4A16 one."""
    wl = syn.WORKLOADS[0]
    rng = np.random.default_rng(2)
    g = np.float32(2.0 ** -10)
    T, H, E, k = 4, wl.H, 4, 2
    codes = rng.integers(0, 8, size=(T, H)) * np.where(rng.random((T, H)) < 0.5, -1, 1)
    codes[:, ::16] = 7                                   # magnitude 6 in every block
    sb = 2.0 ** rng.integers(-2, 3, size=(T, H // 16))  # exact E4M3 block scales
    x = (np.sign(codes) * E2M1[np.abs(codes)]) * np.repeat(sb, 16, axis=1) * g
    xb = _bf16(x)
    assert np.array_equal(oracle.bf16_to_f32(xb), x.astype(np.float32))
    qs = [oracle.quant_nvfp4(syn.gen_expert(wl, w, e)) for w in ("gate", "up") for e in range(E)]
    gate = oracle.Bank(oracle.FMT_NVFP4, np.stack([q[0] for q in qs[:E]]), np.stack([q[1] for q in qs[:E]]),
                       np.array([q[2] for q in qs[:E]], np.float32))
    up = oracle.Bank(oracle.FMT_NVFP4, np.stack([q[0] for q in qs[E:]]), np.stack([q[1] for q in qs[E:]]),
                     np.array([q[2] for q in qs[E:]], np.float32))
    ids = np.array([[0, 1], [2, 3], [1, 0], [3, 2]], np.int32)
    off, rs, sr = oracle.permute(ids, E)
    rows = np.arange(T * k)
    h4 = oracle.grouped_swiglu_w4a4(xb, off, rs, k, gate, up, np.full(E, g, np.float32), rows)
    h16 = oracle.grouped_swiglu(xb, off, rs, k, gate, up, rows)
    assert np.array_equal(h4, h16)


def test_act_quant_saturates():
    x = _bf16(np.full((1, 16), 10.0))
    packed, scales, xq = oracle.act_quant_nvfp4(x, 1e-3)     # 10 / (6 * 1e-3) > 448
    assert scales[0, 0] == 0x7E
    assert np.all(packed == 0x77)                              # +6 everywhere
    assert np.allclose(xq, 6 * 448 * 1e-3, rtol=1e-6)


def _w4a4_problem(seed=0):
    wl = syn.WORKLOADS[0]
    x = syn.gen_x(wl, seed)
    Wr = syn.gen_router(wl, seed)
    banks = {}
    for which in ("gate", "up", "down"):
        qs = [oracle.quant_nvfp4(syn.gen_expert(wl, which, e, seed)) for e in range(wl.E)]
        banks[which] = oracle.Bank(oracle.FMT_NVFP4, np.stack([q[0] for q in qs]), np.stack([q[1] for q in qs]),
                                   np.array([q[2] for q in qs], np.float32))
    rng = np.random.default_rng(seed + 5)
    # static activation scales: the inputs' amax / (6 * 448) (x is N(0, 1); h stays well below 1),
    # varied per expert so that each expert's own scale is exercised
    in_gu = (4.0 / (6 * 448) * rng.uniform(0.8, 1.25, wl.E)).astype(np.float32)
    in_dn = (0.02 / (6 * 448) * rng.uniform(0.8, 1.25, wl.E)).astype(np.float32)
    sh = tuple(oracle.Bank(oracle.FMT_BF16, syn.gen_shared(wl, w, seed)[None]) for w in ("gate", "up", "down"))
    return wl, x, Wr, banks, in_gu, in_dn, sh


def test_w4a4_layer_matches_dense_mixture():
    wl, x, Wr, banks, in_gu, in_dn, sh = _w4a4_problem()
    ids, w = oracle.route(x, Wr, None, wl.k)
    y = oracle.moe_forward_w4a4(x, ids, w, banks["gate"], banks["up"], banks["down"], in_gu, in_dn, shared=sh)
    xf = torch.from_numpy(oracle.bf16_to_f32(x)).double()
    T = x.shape[0]
    ref = torch.zeros(T, wl.H, dtype=torch.float64)
    for e in range(wl.E):
        Wg, Wu, Wd = (torch.from_numpy(oracle.dequant_expert(banks[n], e)).double() for n in ("gate", "up", "down"))
        xq = torch.from_numpy(oracle.act_quant_nvfp4(x, in_gu[e])[2]).double()
        h = torch.nn.functional.silu(xq @ Wg.T) * (xq @ Wu.T)
        hq = torch.from_numpy(oracle.act_quant_nvfp4(_bf16(h.numpy()), in_dn[e])[2]).double()
        m = torch.from_numpy(np.array([float(w[t][list(ids[t]).index(e)]) if e in ids[t] else 0.0
                                       for t in range(T)]))
        ref += m[:, None] * (hq @ Wd.T)
    Sg, Su, Sd = (torch.from_numpy(oracle.dequant_expert(b, 0)).double() for b in sh)
    ref += (torch.nn.functional.silu(xf @ Sg.T) * (xf @ Su.T)) @ Sd.T
    ref = ref.numpy()
    assert np.max(np.abs(y - ref)) <= 1e-10 * np.max(np.abs(ref))
    # and it differs from W4A16 by a quantisation-sized amount, not by nothing
    y16 = oracle.moe_forward(x, ids, w, banks["gate"], banks["up"], banks["down"], shared=sh)
    d = np.max(np.abs(y - y16)) / np.max(np.abs(y16))
    assert 1e-3 < d < 0.5
