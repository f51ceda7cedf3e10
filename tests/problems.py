"""Problem builders shared by the GPU parity tests.

Inputs come from weight_only_bit_route_b200.synthetic (seeded); packed weights
come either from the oracle's quantisers (small workloads) or, at full size,
from the generator's random codes for the experts the checked tokens touch
(other experts hold zero codes and zero scales).  Nothing here reads a result
of the CUDA library.
"""
import numpy as np
import torch

import oracle
from weight_only_bit_route_b200 import synthetic as syn

FMT = {"int4": oracle.FMT_INT4, "nvfp4": oracle.FMT_NVFP4}


class Problem:
    pass


def _bank_arrays(wl, which, experts, mode, seed):
    """Packed arrays [E, out, ...] for one projection."""
    out, inn = (wl.H, wl.F) if which == "down" else (wl.F, wl.H)
    E = wl.E
    if wl.fmt == "int4":
        packed = np.zeros((E, out, inn // 8), np.int32)
        scales = np.zeros((E, out, inn // 128), np.uint16)
        glob = None
    else:
        packed = np.zeros((E, out, inn // 2), np.uint8)
        scales = np.zeros((E, out, inn // 16), np.uint8)
        glob = np.zeros(E, np.float32)
    for e in experts:
        if mode == "quantised":
            w = syn.gen_expert(wl, which, e, seed)
            if wl.fmt == "int4":
                packed[e], scales[e] = oracle.quant_int4_g128(w)
            else:
                packed[e], scales[e], glob[e] = oracle.quant_nvfp4(w)
        else:
            p, s, g = syn.gen_random_codes(wl, which, e, seed)
            packed[e], scales[e] = p, s
            if glob is not None:
                glob[e] = g
    return packed, scales, glob


def build(cfg, mode="quantised", T=None, seed=0, experts=None, shared=None, check_tokens=None):
    """Inputs, oracle banks and routing for a workload.

    mode: "quantised" (oracle quantiser on every listed expert) or "random"
    (generator codes).  experts: experts to fill (default: those the oracle
    routing selects for check_tokens, or all tokens)."""
    wl = syn.WORKLOADS[cfg] if isinstance(cfg, int) else cfg
    P = Problem()
    P.wl = wl
    P.T = wl.T if T is None else T
    P.x = syn.gen_x(wl, seed, T=P.T)
    P.Wr = syn.gen_router(wl, seed)
    P.bias = syn.gen_bias(wl, seed)
    P.ids, P.w, P.scores = oracle.route(P.x, P.Wr, P.bias, wl.k, want_scores=True)
    P.check_tokens = np.arange(P.T, dtype=np.int32) if check_tokens is None else np.asarray(check_tokens, np.int32)
    if experts is None:
        ex = set(P.ids[P.check_tokens].ravel().tolist())
        # a near-tied token may select its (k+1)-th expert on the GPU: give that expert weights too
        nt = P.check_tokens[near_tie_tokens(P.scores[P.check_tokens], wl.k)]
        for t in nt:
            ex.update(np.argsort(-P.scores[t], kind="stable")[:wl.k + 2].tolist())
        experts = sorted(ex)
    P.experts = experts
    P.banks = {}
    for which in ("gate", "up", "down"):
        packed, scales, glob = _bank_arrays(wl, which, experts, mode, seed)
        P.banks[which] = oracle.Bank(FMT[wl.fmt], packed, scales, glob)
    P.shared = None
    if (wl.shared if shared is None else shared):
        P.shared = tuple(oracle.Bank(oracle.FMT_BF16, syn.gen_shared(wl, w, seed)[None]) for w in ("gate", "up", "down"))
    return P


# ---- device side -----------------------------------------------------------

def dev_bf16(bits, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def dev(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def device_bank(moe, b, device="cuda"):
    if b.fmt == oracle.FMT_INT4:
        return moe.Bank(moe.FMT_INT4_G128, dev(b.packed, device), dev_bf16(b.scales, device))
    if b.fmt == oracle.FMT_NVFP4:
        return moe.Bank(moe.FMT_NVFP4, dev(b.packed, device), dev(b.scales, device), dev(b.global_scale, device))
    return moe.Bank(moe.FMT_BF16, dev_bf16(b.packed, device))


def device_layer(moe, P, device="cuda"):
    banks = [device_bank(moe, P.banks[w], device) for w in ("gate", "up", "down")]
    sh = None if P.shared is None else tuple(device_bank(moe, b, device) for b in P.shared)
    bias = None if P.bias is None else dev(P.bias, device)
    return moe.MoELayer(*banks, router_w=dev(P.Wr, device), top_k=P.wl.k, router_bias=bias, shared=sh)


def bf16_bits(t):
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_ulp(v):
    """One bf16 ulp at |v| (fp64 array)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def layer_tolerance(ref):
    """|gpu - oracle| <= 1e-2 * max|oracle| + one bf16 ulp per element."""
    return 1e-2 * np.max(np.abs(ref)) + bf16_ulp(ref)


def near_tie_tokens(scores, k, eps=1e-5):
    """Tokens whose oracle selection has a near tie: the k-th and (k+1)-th
    scores, or two adjacent selected scores, within eps."""
    s = -np.sort(-scores, axis=1)[:, :k + 1]
    gaps = s[:, :-1] - s[:, 1:]
    return np.nonzero(np.min(gaps, axis=1) <= eps)[0]


def tile_edge_tokens(ids, E, k, nheavy=12, nmaxes=(64, 128, 256), nlight=0):
    """Tokens whose routed rows sit at both edges of every n-tile of the
    nheavy most loaded experts (and the nlight least loaded non-empty ones),
    for the balanced row partitions of the grouped GEMM at each tile height
    in nmaxes (n rows in ceil(n / nmax) tiles of ceil(n / ntile) rows)."""
    off, rs, _ = oracle.permute(ids, E)
    cnt = np.diff(off)
    order = np.argsort(-cnt, kind="stable")
    chosen = list(order[:nheavy])
    if nlight:
        chosen += [e for e in order[::-1] if cnt[e] > 0][:nlight]
    rows = set()
    for e in chosen:
        n = int(cnt[e])
        for nm in nmaxes:
            nt = -(-n // nm)
            per = -(-n // nt)
            for i in range(nt):
                a = i * per
                b = min(n, a + per) - 1
                rows.update((int(off[e] + a), int(off[e] + b)))
    return sorted(set(int(rs[r]) // k for r in rows))


# ---- comparisons ------------------------------------------------------------

def check_ids(ids_gpu, P, tokens):
    """Exact ids outside near ties; valid selections inside.  Returns the
    near-tie tokens found among `tokens`."""
    k = P.wl.k
    nt = set(near_tie_tokens(P.scores[tokens], k).tolist())
    flipped = []
    for i, t in enumerate(tokens):
        if i in nt:
            s = P.scores[t]
            kth = -np.sort(-s)[k - 1]
            sel = ids_gpu[i]
            assert len(set(sel.tolist())) == k
            assert np.all(s[sel] >= kth - 1e-5), (t, sel)
            if not np.array_equal(sel, P.ids[t]):
                flipped.append(int(t))
        else:
            assert np.array_equal(ids_gpu[i], P.ids[t]), (t, ids_gpu[i], P.ids[t])
    return nt, flipped


def layer_check(P, y_gpu, tokens, ids_gpu, w_gpu):
    """Every listed token against the oracle.  ids_gpu / w_gpu: the GPU's routing
    of those tokens.  A near-tied token is recomputed in the oracle with the
    GPU's ids and weights (either selection is a valid top-k), so its output is
    checked too."""
    nt, flipped = check_ids(ids_gpu, P, tokens)
    ids = P.ids.copy()
    w = P.w.copy()
    for i in nt:
        ids[tokens[i]] = ids_gpu[i]
        w[tokens[i]] = w_gpu[i]
    ref = oracle.moe_forward(P.x, ids, w, P.banks["gate"], P.banks["up"], P.banks["down"],
                             shared=P.shared, tokens=tokens)
    got = oracle.bf16_to_f32(y_gpu[tokens]).astype(np.float64)
    tol = layer_tolerance(ref)
    err = np.abs(got - ref)
    assert np.all(err <= tol), f"max err {err.max()} (tol scale {1e-2 * np.max(np.abs(ref))})"
    return len(nt), len(flipped), float(err.max() / np.max(np.abs(ref)))
