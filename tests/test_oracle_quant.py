"""Pins for the oracle's quantisers and dequantisers.

int4: "Step-5-Preview-Int4-g128", Recipe (RTN, seventeen clip ratios from 0.60 to 1.00,
bf16 scales, error table) and Tensor layout.  NVFP4:
"Step-5-Preview-NVFP4-Local", Modifications item 2, Format, Layers 88-90
(NVFP4 weight NMSE) and Fidelity (packed matrices decode exactly to the
quantiser's output; independent decoder).
"""
import os

import numpy as np
import torch

import oracle
from weight_only_bit_route_b200 import synthetic as syn

GOLD = os.path.join(os.path.dirname(__file__), "golden")
E2M1_TABLE = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float32)


def _read_golden(name):
    d = {}
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        d[key] = vals
    return d


def _bf16(a):
    return syn.to_bf16_bits(np.asarray(a, np.float32))


# ---- independent decoders (numpy bit operations + library conversions) ----

def np_decode_int4(packed, scales):
    p = packed.view(np.uint32)
    rows, words = p.shape
    nib = np.stack([(p >> (4 * j)) & 0xF for j in range(8)], axis=-1).reshape(rows, words * 8)
    q = nib.astype(np.int32) - 8
    s = torch.from_numpy(scales.view(np.int16)).view(torch.bfloat16).float().numpy()
    return q.astype(np.float32) * np.repeat(s, 128, axis=1), q


def np_decode_nvfp4(packed, scales, g):
    lo = packed & 0xF
    hi = packed >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(packed.shape[0], packed.shape[1] * 2)
    mag = E2M1_TABLE[codes & 7]
    val = np.where(codes & 8, -mag, mag).astype(np.float32)
    sb = torch.from_numpy(scales).view(torch.float8_e4m3fn).float().numpy()
    return (val * np.repeat(sb, 16, axis=1)) * np.float32(g), codes


# ---- int4 -----------------------------------------------------------------

def test_int4_golden_packing_order():
    gd = _read_golden("int4_pack_order.txt")
    qa = (np.arange(128) % 16) - 8
    w = _bf16(qa * 2.0 ** -6)[None, :]
    packed, scales, ri = oracle.quant_int4_g128(w, want_ratio=True)
    assert scales[0, 0] == int(gd["caseA_scale_bits"][0], 16)
    assert ri[0, 0] == int(gd["caseA_ratio_index"][0])
    want = np.array([int(v, 16) for v in gd["caseA_words"]], np.uint64).astype(np.uint32)
    assert np.array_equal(packed[0].view(np.uint32), want)
    assert np.array_equal(oracle.dequant_int4_g128(packed, scales), oracle.bf16_to_f32(w))

    qb = (np.arange(128) % 15) - 7
    w = _bf16(qb * 2.0 ** -6)[None, :]
    packed, scales, ri = oracle.quant_int4_g128(w, want_ratio=True)
    assert scales[0, 0] == int(gd["caseB_scale_bits"][0], 16)
    assert ri[0, 0] == int(gd["caseB_ratio_index"][0])
    assert np.array_equal(oracle.dequant_int4_g128(packed, scales), oracle.bf16_to_f32(w))


def test_int4_roundtrip_exact_and_independent_decoder():
    wl = syn.WORKLOADS[0]
    w = syn.gen_expert(wl, "gate", 3)          # [256, 1024]
    packed, scales, q = oracle.quant_int4_g128(w, want_q=True)
    deq = oracle.dequant_int4_g128(packed, scales)
    ref, qdec = np_decode_int4(packed, scales)
    assert np.array_equal(qdec, q.astype(np.int32))           # packed codes are the quantiser's codes
    assert np.array_equal(deq, ref)                            # bit-exact decode
    s = oracle.bf16_to_f32(scales)
    assert np.array_equal(deq, q.astype(np.float32) * np.repeat(s, 128, axis=1))


def _candidate_errors(wf, amax):
    """Brute force over the 17 candidates, fp64 error (numpy + torch bf16)."""
    errs, scales = [], []
    for i in range(17):
        r = np.float32(24 + i) / np.float32(40)
        sf = np.float32(np.float32(r * amax) / np.float32(7))
        s = oracle.bf16_to_f32(_bf16([sf]))[0]
        q = np.clip(np.rint(wf.astype(np.float64) / np.float64(s)), -8, 7)
        errs.append(float(np.sum((q * np.float64(s) - wf) ** 2)))
        scales.append(s)
    return np.array(errs), np.array(scales)


def test_int4_clip_choice_is_best_candidate():
    rng = np.random.default_rng(5)
    w = _bf16(rng.standard_normal((16, 1024)).astype(np.float32) * 0.02)
    # add a few outlier groups so clipping matters
    w[0, :128] = _bf16(rng.standard_normal(128).astype(np.float32) * 0.02 * np.where(np.arange(128) == 5, 20, 1))
    packed, scales, ri = oracle.quant_int4_g128(w, want_ratio=True)
    wf = oracle.bf16_to_f32(w)
    s_all = oracle.bf16_to_f32(scales)
    for r in range(w.shape[0]):
        for g in range(w.shape[1] // 128):
            grp = wf[r, g * 128:(g + 1) * 128]
            errs, cands = _candidate_errors(grp, np.float32(np.max(np.abs(grp))))
            chosen = s_all[r, g]
            assert chosen in cands
            assert chosen == cands[ri[r, g]]
            # fp32 accumulation in the oracle vs fp64 here: allow rounding-level slack
            assert errs[ri[r, g]] <= errs.min() * (1 + 1e-5) + 1e-30


def test_int4_zero_group():
    w = np.zeros((2, 256), np.uint16)
    packed, scales = oracle.quant_int4_g128(w)
    assert np.all(scales == 0)
    assert np.all(packed.view(np.uint32) == 0x88888888)
    assert np.all(oracle.dequant_int4_g128(packed, scales) == 0)


def _rel_err(wq, w, x):
    return np.linalg.norm((wq - w) @ x) / np.linalg.norm(w @ x)


def test_int4_error_bands_match_pages_table():
    """The page's table: max-abs 11.74 %, clip search 10.11 % (8 experts, Gaussian x).
    Gaussian N(0, 0.02^2) matrices stand in for the real experts."""
    wl = syn.WORKLOADS[1]
    rng = np.random.default_rng(11)
    mats = []
    for which in ("gate", "up", "down", "gate"):
        for e in (7, 200):
            full = syn.gen_expert(wl, which, e)
            mats.append(full[:192])
    max_abs, clip = [], []
    for w in mats:
        wf = oracle.bf16_to_f32(w).astype(np.float64)
        x = rng.standard_normal((w.shape[1], 32))
        p1, s1 = oracle.quant_int4_g128(w, max_abs_only=True)
        p2, s2 = oracle.quant_int4_g128(w)
        e1 = _rel_err(oracle.dequant_int4_g128(p1, s1), wf, x)
        e2 = _rel_err(oracle.dequant_int4_g128(p2, s2), wf, x)
        assert e2 < e1
        max_abs.append(e1)
        clip.append(e2)
    ma, cl = 100 * np.mean(max_abs), 100 * np.mean(clip)
    assert 11.0 <= ma <= 12.5, ma
    assert 9.5 <= cl <= 10.7, cl


# ---- NVFP4 ----------------------------------------------------------------

def test_nvfp4_golden_block():
    gd = _read_golden("nvfp4_block.txt")
    v = np.array([float(a) for a in gd["values"]], np.float32)
    w = _bf16(v * 2.0 ** -4)[None, :]
    packed, scales, g = oracle.quant_nvfp4(w)
    assert g == float(np.float32(0.375) / np.float32(2688))
    assert scales[0, 0] == int(gd["scale_byte"][0], 16)
    assert packed[0].tolist() == [int(b, 16) for b in gd["bytes"]]
    _, codes = np_decode_nvfp4(packed, scales, g)
    assert codes[0].tolist() == [int(c, 16) for c in gd["codes"]]


def test_nvfp4_roundtrip_exact_and_independent_decoder():
    wl = syn.WORKLOADS[0]
    w = syn.gen_expert(wl, "down", 1)           # [1024, 256]
    packed, scales, g = oracle.quant_nvfp4(w)
    deq = oracle.dequant_nvfp4(packed, scales, g)
    ref, codes = np_decode_nvfp4(packed, scales, g)
    assert np.array_equal(deq, ref)
    # global rule and block-scale range
    wf = oracle.bf16_to_f32(w)
    assert g == float(np.float32(np.max(np.abs(wf))) / np.float32(6 * 448))
    assert scales.max() <= 0x7E


def test_nvfp4_codes_are_nearest():
    """Brute force: each code is the nearest of the 16 E2M1 values at the
    block's effective scale e4m3(sb) * g (ties excluded)."""
    rng = np.random.default_rng(3)
    w = _bf16(rng.standard_normal((8, 256)).astype(np.float32) * 0.02)
    packed, scales, g = oracle.quant_nvfp4(w)
    wf = oracle.bf16_to_f32(w).astype(np.float64)
    _, codes = np_decode_nvfp4(packed, scales, g)
    sb = torch.from_numpy(scales).view(torch.float8_e4m3fn).float().numpy()
    eff = np.repeat(np.float32(sb) * np.float32(g), 16, axis=1).astype(np.float64)
    allv = np.concatenate([E2M1_TABLE, -E2M1_TABLE]).astype(np.float64)
    d = np.abs(allv[None, None, :] * eff[..., None] - wf[..., None])
    best = d.min(axis=-1)
    mag = E2M1_TABLE[codes & 7].astype(np.float64)
    got = np.abs(np.where(codes & 8, -mag, mag) * eff - wf)
    assert np.all(got <= best * (1 + 1e-6) + 1e-30)
    # block scales: amax of each block lands within E4M3 rounding of 6 * e4m3(sb) * g
    amax_b = np.abs(wf).reshape(8, 16, 16).max(-1)
    ratio = amax_b / (6 * eff[:, ::16])
    assert np.all(np.abs(ratio - 1) <= 1 / 16 + 1e-6)


def test_nvfp4_zero_matrix_and_zero_block():
    w = np.zeros((2, 32), np.uint16)
    packed, scales, g = oracle.quant_nvfp4(w)
    assert g == 0.0 and np.all(scales == 0) and np.all(packed == 0)
    w = _bf16(np.concatenate([np.zeros(16), np.linspace(-0.1, 0.1, 16)]).astype(np.float32))[None, :]
    packed, scales, g = oracle.quant_nvfp4(w)
    assert scales[0, 0] == 0 and np.all(packed[0, :8] == 0)
    assert np.all(oracle.dequant_nvfp4(packed, scales, g)[0, :16] == 0)


def test_nvfp4_nmse_band_matches_page():
    """NVFP4 weight NMSE 0.903 % on real experts ("Step-5-Preview-NVFP4-Local",
    Layers 88-90); Gaussian N(0, 0.02^2) experts stand in."""
    wl = syn.WORKLOADS[1]
    num = den = 0.0
    for which, e in (("gate", 3), ("up", 9), ("down", 21)):
        w = syn.gen_expert(wl, which, e)[:512]
        packed, scales, g = oracle.quant_nvfp4(w)
        wf = oracle.bf16_to_f32(w).astype(np.float64)
        deq = oracle.dequant_nvfp4(packed, scales, g).astype(np.float64)
        num += np.sum((deq - wf) ** 2)
        den += np.sum(wf ** 2)
    nmse = 100 * num / den
    assert 0.85 <= nmse <= 0.96, nmse


def test_layout_sizes_match_pages():
    """Byte counts that fix the layouts: scales per layer 352 x (2*1536*256 +
    4096*96) bytes, x85 layers = 35,295,068,160 ("Step-5-Preview-NVFP4-Local",
    Size); NVFP4 weights of 3 layers = 9,965,666,304; 18,874,368 params per
    expert ("Step 5 Preview...", Counting the parameters)."""
    E, H, F = 352, 4096, 1536
    scale_bytes = E * (2 * F * (H // 16) + H * (F // 16))
    assert scale_bytes == 415_236_096
    assert 85 * scale_bytes == 35_295_068_160
    assert 3 * E * 3 * F * H // 2 == 9_965_666_304
    assert 3 * F * H == 18_874_368
    # int4 per expert: packed + bf16 scales
    assert 3 * F * H // 2 + 3 * F * H // 128 * 2 == 9_732_096
    # NVFP4 per expert: packed + E4M3 scales + one fp32 weight_scale_2 per projection
    assert 3 * F * H // 2 + 3 * F * H // 16 + 3 * 4 == 10_616_844
