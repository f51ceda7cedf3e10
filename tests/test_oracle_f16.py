"""Pins for the oracle's fp16 input activations ("Step-5-Preview-Spark", At a
glance and Quality: the release runs activations in fp16; bf16 rounding of the
routing input changed far more top-8 sets than fp16)."""
import numpy as np

import oracle
from weight_only_bit_route_b200 import synthetic as syn


def test_f16_decode_exhaustive_vs_numpy():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = codes.view(np.float16).astype(np.float32)
    got = np.array([oracle.f16_to_f32(c) for c in codes], np.float32)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))


def _int4_tiny():
    wl = syn.WORKLOADS[0]
    banks = {}
    for which in ("gate", "up", "down"):
        qs = [oracle.quant_int4_g128(syn.gen_expert(wl, which, e)) for e in range(wl.E)]
        banks[which] = oracle.Bank(oracle.FMT_INT4, np.stack([q[0] for q in qs]), np.stack([q[1] for q in qs]))
    return wl, banks


def test_f16_input_equals_bf16_input_on_values_both_hold():
    """bf16 values inside fp16's normal range are fp16 values too: the same
    numbers given as fp16 bits route and compute identically."""
    wl, banks = _int4_tiny()
    xb = syn.gen_x(wl)
    xf = oracle.bf16_to_f32(xb)
    assert np.all((np.abs(xf) >= 2.0 ** -14) & (np.abs(xf) < 65504))
    xh = xf.astype(np.float16).view(np.uint16)
    assert np.array_equal(xh.view(np.float16).astype(np.float32), xf)
    Wr = syn.gen_router(wl)
    ids_b, w_b, sc_b = oracle.route(xb, Wr, None, wl.k, want_scores=True)
    y_b = oracle.moe_forward(xb, ids_b, w_b, banks["gate"], banks["up"], banks["down"])
    with oracle.x_f16():
        ids_h, w_h, sc_h = oracle.route(xh, Wr, None, wl.k, want_scores=True)
        y_h = oracle.moe_forward(xh, ids_h, w_h, banks["gate"], banks["up"], banks["down"])
    assert np.array_equal(sc_b, sc_h) and np.array_equal(ids_b, ids_h)
    assert np.array_equal(y_b, y_h)


def test_f16_input_is_read_as_f16():
    """fp16 bits that are not bf16 values give the routing of their own values
    (fp64 reference over the decoded fp16 numbers)."""
    wl, _ = _int4_tiny()
    rng = np.random.default_rng(9)
    xh = rng.standard_normal((8, wl.H)).astype(np.float16)
    Wr = syn.gen_router(wl)
    with oracle.x_f16():
        ids, w, sc = oracle.route(xh.view(np.uint16), Wr, None, wl.k, want_scores=True)
    l = xh.astype(np.float64) @ Wr.astype(np.float64).T
    assert np.max(np.abs(sc - 1 / (1 + np.exp(-l)))) < 5e-6
