"""Pins for the oracle's number formats: bf16, E2M1, E4M3.

Independent references: torch's bf16 / float8_e4m3fn conversions (library
routines), the E2M1 value table of the NVFP4 element type, and exhaustive
enumeration.  Source: "Step-5-Preview-NVFP4-Local", Format (E2M1 values, E4M3
block scales) and the int4 page's bf16 scales ("Step-5-Preview-Int4-g128",
Recipe).
"""
import math

import numpy as np
import torch

import oracle

# E2M1 magnitudes of codes 0..7 as listed by the OCP microscaling element type
# that NVFP4 uses; bit 3 is the sign.
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_bf16_rne_matches_torch():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 20000),
        # exact bf16 midpoints: ties must go to the even mantissa
        ((np.arange(2000, dtype=np.uint32) << 16) | 0x8000).view(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38, 1e-40, -1e-40], np.float32),
    ]).astype(np.float32)
    vals = vals[np.isfinite(vals)]
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16_scalar(v) for v in vals], np.uint16)
    assert np.array_equal(got, ref)
    # and back: bf16 -> fp32 is exact widening
    back = oracle.bf16_to_f32(ref)
    assert np.array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_e4m3_decode_exhaustive_vs_torch():
    allb = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = allb.view(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle.e4m3_decode(b) for b in range(256)], np.float32)
    nan_ref = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan_ref)
    assert set(np.nonzero(nan_ref)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(got[~nan_ref], ref[~nan_ref])


def test_e4m3_table_facts():
    pos = [oracle.e4m3_decode(b) for b in range(1, 0x7F)]
    assert len(pos) == 126 and all(v > 0 for v in pos)
    assert all(a < b for a, b in zip(pos, pos[1:]))       # strictly increasing codes
    assert max(pos) == 448.0
    assert min(pos) == 2.0 ** -9
    assert oracle.e4m3_decode(0x00) == 0.0 and math.copysign(1, oracle.e4m3_decode(0x80)) < 0


def test_e4m3_encode_roundtrip_midpoints_and_vs_torch():
    vals = [oracle.e4m3_decode(b) for b in range(0, 0x7F)]
    for b, v in enumerate(vals):
        assert oracle.e4m3_encode(v) == b
    # midpoints go to the even code
    for b in range(0, 0x7E):
        mid = (np.float64(vals[b]) + np.float64(vals[b + 1])) / 2
        if np.float32(mid) != mid:
            continue
        want = b if b % 2 == 0 else b + 1
        assert oracle.e4m3_encode(float(mid)) == want, (b, mid)
    # saturation
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(1e6) == 0x7E
    assert oracle.e4m3_encode(0.0) == 0
    # random values inside the range against torch's RNE cast
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.uniform(0, 448, 3000), np.exp(rng.uniform(np.log(1e-4), np.log(448), 3000))])
    x = x.astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(v) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_e2m1_decode_table():
    for c in range(16):
        mag = E2M1_TABLE[c & 7]
        want = -mag if c & 8 else mag
        got = oracle.e2m1_decode(c)
        assert got == want and math.copysign(1, got) == (-1 if c & 8 else 1)


def test_e2m1_encode_nearest_ties_even_saturating():
    for c in range(16):
        if c == 8:
            continue
        assert oracle.e2m1_encode(oracle.e2m1_decode(c)) == c
    # midpoints between neighbours -> code with zero mantissa bit
    for lo in range(7):
        mid = (E2M1_TABLE[lo] + E2M1_TABLE[lo + 1]) / 2
        want = lo if lo % 2 == 0 else lo + 1
        assert oracle.e2m1_encode(mid) == want
        assert oracle.e2m1_encode(-mid) == (8 | want)
    assert oracle.e2m1_encode(7.0) == 7 and oracle.e2m1_encode(1e9) == 7
    assert oracle.e2m1_encode(-100.0) == 0xF
    # brute-force nearest on a dense sweep
    for v in np.linspace(-7, 7, 2801):
        c = oracle.e2m1_encode(float(v))
        d = abs(oracle.e2m1_decode(c) - v)
        assert all(d <= abs(s * m - v) + 1e-12 for m in E2M1_TABLE for s in (1, -1))
