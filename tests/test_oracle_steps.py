"""Pins for the oracle's per-step definitions: grouped gate/up + SwiGLU, grouped
down with the routing weight, and the unpermute + combine.

Layer: "Step 5 Preview: 92 narrow layers...", The shape (each token is its
shared SwiGLU expert plus its routed SwiGLU experts, weighted).  Storage:
"Step-5-Preview-Int4-g128", Recipe / Tensor layout; "Step-5-Preview-NVFP4-Local",
Format.

Three independent references:
  1. a hand-derived two-expert case (tests/golden/two_expert_composition.txt)
     whose every intermediate has a closed form;
  2. the chain route -> permute -> grouped_swiglu -> bf16 -> grouped_down ->
     bf16 -> combine (shared expert through the same calls with E = 1) against
     the brute-force dense mixture over ALL experts, within a bound derived
     from the two bf16 roundings (each at most 2^-8 relative);
  3. special cases: a dropped slot (row -1) adds nothing; the routing weight is
     taken by slot, so permuting rows inside an expert permutes the outputs.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from weight_only_bit_route_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "two_expert_composition.txt")
U_BF16 = 2.0 ** -8          # unit roundoff of bf16 round-to-nearest-even


def _bf16(a):
    return syn.to_bf16_bits(np.asarray(a, np.float32))


def _f(bits):
    return oracle.bf16_to_f32(bits).astype(np.float64)


def _pack_int4(q):
    """q int [rows, cols] in [-8, 7] -> int32 words, element 8c+j in bits 4j..4j+3, nibble q+8."""
    rows, cols = q.shape
    u = (q + 8).astype(np.uint32).reshape(rows, cols // 8, 8)
    words = np.zeros((rows, cols // 8), np.uint32)
    for j in range(8):
        words |= u[:, :, j] << np.uint32(4 * j)
    return words.view(np.int32)


def _golden_case():
    H = F = 128
    hh = np.arange(H)
    x = np.stack([(hh % 5) - 2, (3 * hh % 7) - 3]).astype(np.float64)
    ids = np.array([[1, 0], [0, 1]], np.int32)
    tw = np.array([[0.75, 0.25], [0.5, 0.5]], np.float32)

    def bank(qs, scales):
        packed = np.stack([_pack_int4(q) for q in qs])
        sc = np.stack([np.full((q.shape[0], 1), s, np.float32) for q, s in zip(qs, scales)])
        return oracle.Bank(oracle.FMT_INT4, packed, _bf16(sc))

    eye = np.eye(F, H, dtype=np.int64)
    shift1 = np.roll(eye, 1, axis=1)                  # row f -> column f+1
    shift3 = np.roll(np.eye(H, F, dtype=np.int64), 3, axis=1)
    gate = bank([1 * eye, 2 * eye], [0.25, 0.25])
    up = bank([shift1, -shift1], [0.5, 0.5])
    down = bank([eye, -2 * shift3], [1.0, 0.5])
    return x, ids, tw, gate, up, down


def _golden_values():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, t, i, v = line.split()
        vals[(name, int(t), int(i))] = float(v)
    return vals


def _silu(v):
    return v / (1.0 + np.exp(-v))


def test_golden_two_expert_composition():
    x, ids, tw, gate, up, down = _golden_case()
    xb = _bf16(x)
    assert np.array_equal(_f(xb), x)                  # small integers: exact in bf16
    T, k = ids.shape
    off, rs, sr = oracle.permute(ids, 2)
    assert off.tolist() == [0, 2, 4] and rs.tolist() == [1, 2, 0, 3] and sr.tolist() == [2, 0, 1, 3]

    # gate/up + SwiGLU: every element against its closed form
    h = oracle.grouped_swiglu(xb, off, rs, k, gate, up, np.arange(T * k))
    xn = np.roll(x, -1, axis=1)                       # x[t, f+1]
    h_cf = {0: _silu(x / 4) * (0.5 * xn), 1: _silu(x / 2) * (-0.5 * xn)}
    for r in range(T * k):
        e = 0 if r < off[1] else 1
        t = rs[r] // k
        assert np.allclose(h[r], h_cf[e][t], rtol=1e-14, atol=0)

    # down with the routing weight taken by slot, from the bf16-rounded h
    hb = _bf16(h)
    y_perm = oracle.grouped_down(hb, off, rs, tw.ravel(), down, np.arange(T * k))
    for r in range(T * k):
        e = 0 if r < off[1] else 1
        s = rs[r]
        hr = _f(hb[r])
        d = hr if e == 0 else -np.roll(hr, -3)        # D_1[i] = -h_1[i + 3]
        assert np.array_equal(y_perm[r], np.float64(tw.ravel()[s]) * d)

    # combine: shared + the slots' rows (two bf16 terms and the shared term sum exactly in fp64)
    ypb = _bf16(y_perm)
    sh = _bf16(x / 8)
    y = oracle.combine(ypb, sr, T, k, sh)
    want = _f(sh) + _f(ypb[sr[0::2]]) + _f(ypb[sr[1::2]])
    assert np.array_equal(y, want)

    # the hand-worked values (no intermediate rounding; the chain rounds twice to bf16)
    for (name, t, i), v in _golden_values().items():
        if name == "y":
            assert abs(y[t, i] - v) <= 4 * U_BF16 * (abs(v) + 0.25), (t, i, y[t, i], v)
            exact = float(x[t, i]) / 8 + sum(
                float(tw[t, j]) * (h_cf[0][t, i] if ids[t, j] == 0 else -h_cf[1][t, (i + 3) % 128]) for j in range(k))
            assert math.isclose(exact, v, rel_tol=1e-14)
        else:
            e = int(name[1])
            assert math.isclose(h_cf[e][t, i], v, rel_tol=1e-14)


def test_combine_skips_dropped_slot():
    """A slot with row -1 (an id the bucketing dropped) contributes nothing."""
    rng = np.random.default_rng(3)
    T, k, H = 3, 2, 16
    yp = _bf16(rng.standard_normal((T * k, H)))
    sr = np.array([0, 1, -1, 2, 3, 4], np.int32)
    y = oracle.combine(yp, sr, T, k)
    assert np.array_equal(y[1], _f(yp[2]))
    assert np.array_equal(y[0], _f(yp[0]) + _f(yp[1]))


def test_down_weight_is_taken_by_slot():
    """Reversing the rows of one expert (and their slots) reverses its outputs:
    the weight follows the slot, not the row position."""
    rng = np.random.default_rng(5)
    wl = syn.WORKLOADS[0]
    F, H, E = wl.F, wl.H, 2
    qd = [oracle.quant_int4_g128(syn.gen_expert(wl, "down", e)) for e in range(E)]
    down = oracle.Bank(oracle.FMT_INT4, np.stack([q[0] for q in qd]), np.stack([q[1] for q in qd]))
    hb = _bf16(rng.standard_normal((5, F)) * 0.1)
    off = np.array([0, 3, 5], np.int32)
    rs = np.array([4, 0, 2, 1, 3], np.int32)
    tw = np.array([0.1, 0.2, 0.3, 0.4, 0.5], np.float32)
    y = oracle.grouped_down(hb, off, rs, tw, down, np.arange(5))
    perm = np.array([2, 1, 0, 4, 3])
    y2 = oracle.grouped_down(hb[perm], off, rs[perm], tw, down, np.arange(5))
    assert np.array_equal(y2, y[perm])
    y1 = oracle.grouped_down(hb, off, rs, None, down, np.arange(5))
    assert np.allclose(y, y1 * tw[rs][:, None].astype(np.float64), rtol=1e-15, atol=0)


def _dequant_all(bank):
    return [torch.from_numpy(oracle.dequant_expert(bank, e)).double() for e in range(bank.E)]


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_step_chain_matches_dense_mixture(fmt):
    """route -> permute -> grouped_swiglu -> bf16 -> grouped_down -> bf16 -> combine,
    with the shared expert through the same calls (E = 1, offsets {0, T},
    row i at slot i*k), equals the dense mixture over all experts within the
    bound the two bf16 roundings imply."""
    wl = syn.WORKLOADS[0]
    T, H, F, E, k = wl.T, wl.H, wl.F, wl.E, wl.k
    x = syn.gen_x(wl)
    Wr = syn.gen_router(wl)
    banks = {}
    for which in ("gate", "up", "down"):
        mats = [syn.gen_expert(wl, which, e) for e in range(E)]
        if fmt == "int4":
            qs = [oracle.quant_int4_g128(m) for m in mats]
            banks[which] = oracle.Bank(oracle.FMT_INT4, np.stack([q[0] for q in qs]), np.stack([q[1] for q in qs]))
        else:
            qs = [oracle.quant_nvfp4(m) for m in mats]
            banks[which] = oracle.Bank(oracle.FMT_NVFP4, np.stack([q[0] for q in qs]), np.stack([q[1] for q in qs]),
                                       np.array([q[2] for q in qs], np.float32))
    sh = tuple(oracle.Bank(oracle.FMT_BF16, syn.gen_shared(wl, w)[None]) for w in ("gate", "up", "down"))

    ids, tw = oracle.route(x, Wr, None, k)
    off, rs, sr = oracle.permute(ids, E)
    R = T * k
    h = oracle.grouped_swiglu(x, off, rs, k, banks["gate"], banks["up"], np.arange(R))
    hb = _bf16(h)
    yp = oracle.grouped_down(hb, off, rs, tw.ravel(), banks["down"], np.arange(R))
    ypb = _bf16(yp)
    so = np.array([0, T], np.int32)
    srs = (np.arange(T) * k).astype(np.int32)
    hs = oracle.grouped_swiglu(x, so, srs, k, sh[0], sh[1], np.arange(T))
    hsb = _bf16(hs)
    ys = oracle.grouped_down(hsb, so, srs, None, sh[2], np.arange(T))
    ysb = _bf16(ys)
    y = oracle.combine(ypb, sr, T, k, ysb)

    # brute force: every expert on every token, masked by the routing weights
    xf = torch.from_numpy(_f(x))
    Wg, Wu, Wd = (_dequant_all(banks[w]) for w in ("gate", "up", "down"))
    Sg, Su, Sd = (torch.from_numpy(oracle.dequant_expert(b, 0)).double() for b in sh)
    m = torch.zeros(T, E, dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            m[t, ids[t, j]] = float(tw[t, j])
    ref = torch.zeros(T, H, dtype=torch.float64)
    bound = torch.zeros(T, H, dtype=torch.float64)
    for e in range(E):
        he = torch.nn.functional.silu(xf @ Wg[e].T) * (xf @ Wu[e].T)
        de = he @ Wd[e].T
        ref += m[:, e:e + 1] * de
        # rounding h to bf16 moves the down output by at most u * |Wd| |h|; rounding
        # y_perm to bf16 moves each slot's row by at most u * |w * (Wd h)|
        bound += m[:, e:e + 1] * (U_BF16 * (he.abs() @ Wd[e].abs().T) * (1 + U_BF16) + U_BF16 * de.abs() * (1 + 2 * U_BF16))
    hsh = torch.nn.functional.silu(xf @ Sg.T) * (xf @ Su.T)
    dsh = hsh @ Sd.T
    ref += dsh
    bound += U_BF16 * (hsh.abs() @ Sd.abs().T) * (1 + U_BF16) + U_BF16 * dsh.abs() * (1 + 2 * U_BF16)
    ref, bound = ref.numpy(), bound.numpy()
    err = np.abs(y - ref)
    assert np.all(err <= bound + 1e-12 * np.max(np.abs(ref))), float(np.max(err - bound))
    # the bound is tight enough to see a slipped routing weight: swapping two slots' weights breaks it
    tw_bad = tw.copy()
    tw_bad[:, [0, 1]] = tw_bad[:, [1, 0]]
    yp_bad = _bf16(oracle.grouped_down(hb, off, rs, tw_bad.ravel(), banks["down"], np.arange(R)))
    y_bad = oracle.combine(yp_bad, sr, T, k, ysb)
    assert np.any(np.abs(y_bad - ref) > bound + 1e-12 * np.max(np.abs(ref)))
