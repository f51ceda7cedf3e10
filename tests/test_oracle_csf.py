"""Pins for the oracle's compressed scale format (CSF) encoder and decoder.

"Step-5-Preview-NVFP4-Local", Format: fixed U8 [E, R/16, 16 * (1 + C/2)] (each
slab of 16 rows: their bases, then their 4-bit codes, lower nibble first),
exceptions U32 (row * C + col) | byte << 24, expert by expert in increasing
position, starts I64 [E + 1]; a byte is base + code unless an exception
replaces it; a row's base is the smallest value in 0..240 whose 16-value window
holds the largest number of the row's bytes.  Size: the CSF planes of layers 3-87 take 51.44 % of the raw
block scales.  Fidelity: a second decoder, written separately, recovers from
each CSF tensor exactly the scale bytes it was made from.
"""
import os

import numpy as np

import oracle
from weight_only_bit_route_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "csf_slab.txt")


def _golden():
    sec, out = None, {}
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if not line:
            continue
        if line in ("scales", "fixed", "exceptions", "starts"):
            sec = line
            out[sec] = []
            continue
        out[sec].extend(line.split())
    sc = np.array([int(v, 16) for v in out["scales"]], np.uint8).reshape(1, 16, 4)
    fx = np.array([int(v, 16) for v in out["fixed"]], np.uint8).reshape(1, 1, 16 * 3)
    ex = np.array([int(v, 16) for v in out["exceptions"]], np.uint32)
    st = np.array([int(v) for v in out["starts"]], np.int64)
    return sc, fx, ex, st


def _numpy_decode(fixed, exc, starts, R, C):
    """Independent decoder: vectorised slab unpacking, then the exceptions."""
    E = fixed.shape[0]
    sl = fixed.reshape(E, R // 16, 16 * (1 + C // 2))
    base = sl[:, :, :16].reshape(E, R).astype(np.int32)
    codes = sl[:, :, 16:].reshape(E, R // 16, 16, C // 2).reshape(E, R, C // 2)
    nib = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(E, R, C).astype(np.int32)
    out = (base[:, :, None] + nib).astype(np.uint8)
    for e in range(E):
        x = exc[starts[e]:starts[e + 1]]
        flat = out[e].reshape(-1)
        flat[(x & 0xFFFFFF).astype(np.int64)] = (x >> 24).astype(np.uint8)
    return out


def _brute_base(row):
    counts = [np.sum((row >= b) & (row <= b + 15)) for b in range(241)]
    return int(np.argmax(counts))          # argmax returns the first (lowest) maximum


def test_golden_slab():
    sc, fx, ex, st = _golden()
    f, e, s = oracle.csf_encode(sc)
    assert np.array_equal(f, fx)
    assert np.array_equal(e, ex)
    assert np.array_equal(s, st)
    assert np.array_equal(oracle.csf_decode(fx, ex, st, 16, 4), sc)


def test_row_base_is_lowest_best_window():
    rng = np.random.default_rng(1)
    E, R, C = 2, 32, 96
    sc = rng.integers(0, 256, size=(E, R, C), dtype=np.uint8)
    sc[0, 0] = 250                         # constant rows: the window must start at 235
    sc[0, 1] = 0
    sc[1, :8] = rng.integers(0x30, 0x50, size=(8, C), dtype=np.uint8)   # two binades of E4M3 scales
    f, e, s = oracle.csf_encode(sc)
    bases = f.reshape(E, R // 16, -1)[:, :, :16].reshape(E, R)
    for ee in range(E):
        for r in range(R):
            assert bases[ee, r] == _brute_base(sc[ee, r]), (ee, r)
    assert bases[0, 0] == 235 and bases[0, 1] == 0


def test_roundtrip_and_independent_decoder():
    rng = np.random.default_rng(2)
    for E, R, C in ((3, 32, 96), (2, 48, 256), (1, 16, 2)):
        sc = rng.integers(0, 256, size=(E, R, C), dtype=np.uint8)
        f, e, s = oracle.csf_encode(sc)
        assert np.array_equal(oracle.csf_decode(f, e, s, R, C), sc)
        assert np.array_equal(_numpy_decode(f, e, s, R, C), sc)
        # exceptions: exactly the bytes outside their row's window, row-major, positions in range
        bases = f.reshape(E, R // 16, -1)[:, :, :16].reshape(E, R).astype(np.int32)
        outside = (sc < bases[:, :, None]) | (sc > bases[:, :, None] + 15)
        assert np.array_equal(np.diff(s), outside.reshape(E, -1).sum(1))
        for ee in range(E):
            x = e[s[ee]:s[ee + 1]]
            assert np.all(np.diff(x & 0xFFFFFF) > 0)
            assert np.all((x & 0xFFFFFF) < R * C)


def test_nvfp4_scales_roundtrip_and_per_expert_form():
    """Block scales from the NVFP4 quantiser at the gate/up (C = 256) and down
    (C = 96) widths; one expert encoded alone equals its slice of the fused
    encoding (its slab rows, and its span of the exceptions as starts delimits it)."""
    wl = syn.WORKLOADS[0]
    for which, R, C in (("gate", 64, 256), ("down", 32, 96)):
        mats = []
        for e in range(3):
            w = syn.gen_expert(wl, which, e)[:R]
            if w.shape[1] != C * 16:
                w = np.tile(w, (1, (C * 16) // w.shape[1] + 1))[:, :C * 16]
            mats.append(oracle.quant_nvfp4(w)[1])
        sc = np.stack(mats)
        f, e, s = oracle.csf_encode(sc)
        assert np.array_equal(oracle.csf_decode(f, e, s, R, C), sc)
        for ee in range(3):
            f1, e1, s1 = oracle.csf_encode(sc[ee:ee + 1])
            assert np.array_equal(f1[0], f[ee])
            assert np.array_equal(e1, e[s[ee]:s[ee + 1]])


def test_sizes_match_the_pages():
    """Fixed plane E * R * (1 + C/2) bytes and starts 8 * (E + 1) per tensor.
    For the pages' shapes (E = 352; gate and up R = 1536, C = 256; down R = 4096,
    C = 96) the rest of each CSF total in the Size table is a whole number of
    4-byte exceptions, and the total is 51.44 % of the raw scales."""
    E = 352
    shapes = [(1536, 256), (1536, 256), (4096, 96)]
    fixed = sum(E * R * (1 + C // 2) for R, C in shapes)
    starts = 3 * 8 * (E + 1)
    raw = sum(E * R * C for R, C in shapes)
    assert raw == 415_236_096
    for layers, total in ((85, 18_154_837_272), (3, 643_637_016)):
        rest = total - layers * (fixed + starts)
        assert rest > 0 and rest % 4 == 0
        assert rest // 4 < 0.01 * layers * raw      # a small share of the bytes are exceptions
    assert round(100 * 18_154_837_272 / 35_295_068_160, 2) == 51.44
    assert 85 * raw == 35_295_068_160
