"""Pins for the oracle's router, bucketing and layer forward.

Router: "Step-5-Preview-Spark", At a glance (352 experts, top-8, sigmoid
router).  Layer: "Step 5 Preview: 92 narrow layers...", The shape (8 routed
SwiGLU experts of width 1536 plus one shared expert).  Token independence
follows the causality check pattern of "Step-5-Preview-NVFP4-Local", Fidelity.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_bit_route_b200 import synthetic as syn


def _bf16(a):
    return syn.to_bf16_bits(np.asarray(a, np.float32))


def _tiny_problem(wl, fmt="int4", shared=False, seed=0, T=None):
    T = wl.T if T is None else T
    x = syn.gen_x(wl, seed, T=T)
    Wr = syn.gen_router(wl, seed)
    banks = {}
    for which in ("gate", "up", "down"):
        mats = [syn.gen_expert(wl, which, e, seed) for e in range(wl.E)]
        if fmt == "int4":
            qs = [oracle.quant_int4_g128(m) for m in mats]
            banks[which] = oracle.Bank(oracle.FMT_INT4, np.stack([q[0] for q in qs]), np.stack([q[1] for q in qs]))
        else:
            qs = [oracle.quant_nvfp4(m) for m in mats]
            banks[which] = oracle.Bank(oracle.FMT_NVFP4, np.stack([q[0] for q in qs]), np.stack([q[1] for q in qs]),
                                       np.array([q[2] for q in qs], np.float32))
    sh = None
    if shared:
        sh = tuple(oracle.Bank(oracle.FMT_BF16, syn.gen_shared(wl, w, seed)[None]) for w in ("gate", "up", "down"))
    return x, Wr, banks, sh


# ---- router ---------------------------------------------------------------

def test_router_zero_input():
    """x = 0, no bias: every score is sigmoid(0) = 0.5, so ids are 0..7 (ties to
    the lower id) and the renormalised weights are exactly 1/8."""
    x = np.zeros((4, 256), np.uint16)
    Wr = np.random.default_rng(0).standard_normal((32, 256)).astype(np.float32)
    ids, w, sc = oracle.route(x, Wr, None, 8, want_scores=True)
    assert np.all(sc == 0.5)
    assert np.array_equal(ids, np.tile(np.arange(8), (4, 1)))
    assert np.all(w == np.float32(0.125))


def test_router_huge_bias_forces_expert():
    wl = syn.WORKLOADS[0]
    x = syn.gen_x(wl)
    Wr = syn.gen_router(wl)
    bias = np.zeros(wl.E, np.float32)
    bias[13] = 50.0
    ids, w = oracle.route(x, Wr, bias, 8)
    assert np.all(ids[:, 0] == 13)
    ids0, _, sc0 = oracle.route(x, Wr, None, 8, want_scores=True)
    for t in range(wl.T):
        order = [e for e in np.argsort(-sc0[t], kind="stable") if e != 13][:7]
        assert ids[t, 1:].tolist() == order


def test_router_vs_fp64_library_topk():
    """Independent reference: torch fp64 matmul + sigmoid + topk.  Tokens whose
    selection has a near tie (adjacent scores within 1e-5) are excluded."""
    wl = syn.WORKLOADS[1]
    x = syn.gen_x(wl, T=64)
    Wr = syn.gen_router(wl)
    ids, w, sc = oracle.route(x, Wr, None, 8, want_scores=True)
    xf = torch.from_numpy(oracle.bf16_to_f32(x)).double()
    s = torch.sigmoid(xf @ torch.from_numpy(Wr).double().T)
    top = torch.topk(s, 9, dim=1)
    checked = 0
    for t in range(x.shape[0]):
        v = top.values[t].numpy()
        if np.min(np.abs(np.diff(v))) <= 1e-5:
            continue
        checked += 1
        assert ids[t].tolist() == top.indices[t, :8].tolist()
        want = v[:8] / v[:8].sum()
        assert np.allclose(w[t], want, rtol=2e-5, atol=0)
    assert checked >= 32
    # The router is defined in fp32: summing H = 4096 products in fp32 leaves an
    # error of order sqrt(H) * 2^-24 * sum|partial| ~ 1e-6 in the logit.
    assert np.max(np.abs(sc - s.numpy())) <= 5e-6


def test_router_invariants():
    wl = syn.WORKLOADS[4]
    x = syn.gen_x(wl, T=256)
    Wr = syn.gen_router(wl)
    b = syn.gen_bias(wl)
    ids, w = oracle.route(x, Wr, b, 8)
    for t in range(ids.shape[0]):
        assert len(set(ids[t].tolist())) == 8
    assert np.all((ids >= 0) & (ids < wl.E))
    assert np.all(np.abs(w.sum(1) - 1) <= 8 * np.finfo(np.float32).eps)
    assert np.all(np.diff(w, axis=1) <= 0)          # listed by descending score


# ---- permute --------------------------------------------------------------

def test_permute_vs_stable_argsort():
    rng = np.random.default_rng(4)
    for T, E in ((1, 8), (37, 32), (300, 352)):
        ids = np.stack([rng.choice(E, 8, replace=False) for _ in range(T)]).astype(np.int32)
        off, rs, sr = oracle.permute(ids, E)
        flat = ids.ravel()
        assert np.array_equal(rs, np.argsort(flat, kind="stable"))
        assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
        assert np.array_equal(sr[rs], np.arange(T * 8))
        assert np.array_equal(rs[sr], np.arange(T * 8))


def test_permute_degenerate():
    ids = np.zeros((0, 8), np.int32)
    off, rs, sr = oracle.permute(ids, 5)
    assert np.all(off == 0) and rs.size == 0
    ids = np.full((6, 1), 3, np.int32)              # every token on one expert
    off, rs, sr = oracle.permute(ids, 5)
    assert off.tolist() == [0, 0, 0, 0, 6, 6] and rs.tolist() == list(range(6))
    with pytest.raises(ValueError):
        oracle.permute(np.array([[7]], np.int32), 5)


# ---- layer ----------------------------------------------------------------

def _dense_mixture(x, ids, w, banks, sh):
    """Brute force over ALL experts: y = ys + sum_e m[t,e] FFN_e(x), m = 0 off
    the token's top-k (torch fp64, dequantised weights)."""
    E = banks["gate"].E
    xf = torch.from_numpy(oracle.bf16_to_f32(x)).double()
    T = xf.shape[0]
    m = torch.zeros(T, E, dtype=torch.float64)
    for t in range(T):
        for j in range(ids.shape[1]):
            m[t, ids[t, j]] += float(w[t, j])
    y = torch.zeros(T, xf.shape[1], dtype=torch.float64)
    for e in range(E):
        Wg = torch.from_numpy(oracle.dequant_expert(banks["gate"], e)).double()
        Wu = torch.from_numpy(oracle.dequant_expert(banks["up"], e)).double()
        Wd = torch.from_numpy(oracle.dequant_expert(banks["down"], e)).double()
        ffn = (torch.nn.functional.silu(xf @ Wg.T) * (xf @ Wu.T)) @ Wd.T
        y += m[:, e:e + 1] * ffn
    if sh is not None:
        Wg, Wu, Wd = (torch.from_numpy(oracle.dequant_expert(b, 0)).double() for b in sh)
        y += (torch.nn.functional.silu(xf @ Wg.T) * (xf @ Wu.T)) @ Wd.T
    return y.numpy()


@pytest.mark.parametrize("fmt,shared", [("int4", False), ("nvfp4", True)])
def test_layer_matches_dense_mixture(fmt, shared):
    wl = syn.WORKLOADS[0]
    x, Wr, banks, sh = _tiny_problem(wl, fmt, shared)
    ids, w = oracle.route(x, Wr, None, 8)
    y = oracle.moe_forward(x, ids, w, banks["gate"], banks["up"], banks["down"], shared=sh)
    ref = _dense_mixture(x, ids, w, banks, sh)
    assert np.max(np.abs(y - ref)) <= 1e-10 * np.max(np.abs(ref))
    # token subset gives the same rows
    sub = np.array([3, 0, 11], np.int32)
    ys = oracle.moe_forward(x, ids, w, banks["gate"], banks["up"], banks["down"], shared=sh, tokens=sub)
    assert np.array_equal(ys, y[sub])


def test_layer_zero_input_gives_zero():
    wl = syn.WORKLOADS[0]
    _, Wr, banks, sh = _tiny_problem(wl, "int4", True)
    x = np.zeros((3, wl.H), np.uint16)
    ids, w = oracle.route(x, Wr, None, 8)
    y = oracle.moe_forward(x, ids, w, banks["gate"], banks["up"], banks["down"], shared=sh)
    assert np.all(y == 0.0)


def test_layer_token_independence():
    """Perturbing tokens after t0 leaves outputs up to t0 bit-identical."""
    wl = syn.WORKLOADS[0]
    x, Wr, banks, _ = _tiny_problem(wl, "int4", False)
    ids, w = oracle.route(x, Wr, None, 8)
    y = oracle.moe_forward(x, ids, w, banks["gate"], banks["up"], banks["down"])
    x2 = x.copy()
    t0 = 6
    x2[t0 + 1:] = syn.gen_x(wl, seed=99)[t0 + 1:]
    ids2, w2 = oracle.route(x2, Wr, None, 8)
    assert np.array_equal(ids2[:t0 + 1], ids[:t0 + 1])
    y2 = oracle.moe_forward(x2, ids2, w2, banks["gate"], banks["up"], banks["down"])
    assert np.array_equal(y2[:t0 + 1], y[:t0 + 1])
    assert not np.array_equal(y2[t0 + 1:], y[t0 + 1:])


def test_layer_thread_count_independence():
    """The thread count is timing control only: one thread and one per host core give bit-identical scores, ids,
    weights and layer outputs (each parallel item is computed by one thread, and no loop reduces across threads)."""
    wl = syn.WORKLOADS[0]
    x, Wr, banks, sh = _tiny_problem(wl, "nvfp4", True)
    outs = []
    try:
        for n in (1, 0):
            oracle.set_threads(n)
            ids, w, sc = oracle.route(x, Wr, None, 8, want_scores=True)
            y = oracle.moe_forward(x, ids, w, banks["gate"], banks["up"], banks["down"], shared=sh)
            outs.append((ids, w, sc, y))
    finally:
        oracle.set_threads(0)
    for a, b in zip(*outs):
        assert np.array_equal(a, b)


def test_zipf_workload_histogram():
    """The skewed workload leaves some experts empty and a few with > 1500 rows
    at T = 8192 (checked on the full token set)."""
    wl = syn.WORKLOADS[4]
    x = syn.gen_x(wl)
    ids, _ = oracle.route(x, syn.gen_router(wl), syn.gen_bias(wl), 8)
    cnt = np.bincount(ids.ravel(), minlength=wl.E)
    assert (cnt == 0).sum() >= 1
    assert (cnt > 1500).sum() >= 2
