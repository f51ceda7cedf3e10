"""The benchmark's algorithmic byte and FLOP counts (the numerators of every roofline fraction it prints),
checked against things other than its own formulas:

- the bytes of one expert are the sizes of the arrays the oracle's quantisers produce for it (packed codes,
  scales and, for NVFP4, one fp32 global scale per projection), at a small shape;
- at the full shape they are the stored layouts ("Step-5-Preview-Int4-g128", Tensor layout: int32 words of 8
  nibbles and a bf16 scale per 128 inputs; "Step-5-Preview-NVFP4-Local", Format: E2M1 pairs in bytes, an E4M3
  scale per 16 inputs, an fp32 weight_scale_2), counted by hand below;
- the FLOPs are the layer's matrix products counted by brute force on a tiny layer (one multiply-add per weight
  and routed row), and the full-size figure is the same count written out.
- the CSF leg's bytes are the encoded planes and the expanded scales of the experts it expands, counted from the
  oracle's encoding of a tiny layer.
"""
import dataclasses

import numpy as np

import bench
import oracle
from weight_only_bit_route_b200 import synthetic as syn


def _quantised_bytes(wl):
    total = 0
    for which in ("gate", "up", "down"):
        m = syn.gen_expert(wl, which, 0)
        if wl.fmt == "int4":
            packed, scales = oracle.quant_int4_g128(m)
            total += packed.nbytes + scales.nbytes
        else:
            packed, scales, _ = oracle.quant_nvfp4(m)
            total += packed.nbytes + scales.nbytes + 4          # the global scale is stored as fp32
    return total


def test_expert_bytes_are_the_quantised_arrays():
    wl = syn.WORKLOADS[0]
    assert wl.fmt == "int4"
    assert bench.expert_bytes(wl) == _quantised_bytes(wl)
    wl4 = dataclasses.replace(wl, fmt="nvfp4")
    assert bench.expert_bytes(wl4) == _quantised_bytes(wl4)


def test_gateup_bytes_are_two_of_the_three_projections():
    """gate, up and down each hold F x H weights, so gate and up are 2/3 of the expert's bytes."""
    for fmt in ("int4", "nvfp4"):
        wl = dataclasses.replace(syn.WORKLOADS[1], fmt=fmt)
        assert 3 * bench.gateup_bytes_per_expert(wl) == 2 * bench.expert_bytes(wl)


def test_full_size_bytes_by_hand():
    H, F, E, T = 4096, 1536, 352, 8
    # int4 g128: per projection F*H/8 int32 words + F*H/128 bf16 scales
    int4_proj = (F * H // 8) * 4 + (F * H // 128) * 2
    assert int4_proj == 3_244_032
    assert bench.expert_bytes(syn.WORKLOADS[1]) == 3 * int4_proj == 9_732_096
    # NVFP4: F*H/2 code bytes + F*H/16 E4M3 scales + one fp32 global
    fp4_proj = F * H // 2 + F * H // 16 + 4
    assert bench.expert_bytes(syn.WORKLOADS[2]) == 3 * fp4_proj == 10_616_844
    # the decode layer with 60 touched experts: experts + BF16 shared expert + fp32 router + x in and y out (bf16)
    want = 60 * 9_732_096 + 3 * F * H * 2 + E * H * 4 + 2 * T * H * 2
    assert bench.layer_bytes(syn.WORKLOADS[1], 60) == want == 627_572_736


def test_layer_flops_brute_force_tiny():
    """Count one multiply-add (2 FLOPs) per weight element per row that passes through it."""
    wl = dataclasses.replace(syn.WORKLOADS[0], T=3, H=128, E=4, F=64, k=2, shared=True)
    gate = np.ones((wl.F, wl.H))
    down = np.ones((wl.H, wl.F))
    router = np.ones((wl.E, wl.H))
    flops = 0
    for _ in range(wl.T):
        flops += 2 * router.size                                   # logits
        for _ in range(wl.k + 1):                                  # k routed experts and the shared one
            flops += 2 * (2 * gate.size) + 2 * down.size           # gate, up, down
    assert bench.layer_flops(wl) == flops


def test_prefill_flops_by_hand():
    H, F, E, k, T = 4096, 1536, 352, 8, 2048
    per_token = k * 2 * 3 * F * H + 2 * 3 * F * H + 2 * E * H
    assert bench.layer_flops(syn.WORKLOADS[3]) == T * per_token
    # the gate/up call alone: 2 projections x 2 FLOPs x F x H per routed row, 8T rows
    assert 2 * 2 * F * H * k * T == 412_316_860_416


def test_csf_expansion_bytes(monkeypatch):
    """The bench's CSF leg counts, per expert expanded, its fixed slab bytes, its exceptions (4 bytes each), its
    pair of starts and the scale bytes it writes.  Run on a tiny layer with the oracle's encoder and decoder
    standing in for the library (the accounting, not the kernels, is under test)."""
    import types

    import torch

    rng = np.random.default_rng(5)
    E, R, C, k = 6, 32, 64, 2
    wl = dataclasses.replace(syn.WORKLOADS[0], T=3, E=E, k=k)
    banks = [types.SimpleNamespace(scales=torch.from_numpy(rng.integers(0x30, 0x50, size=(E, R, C), dtype=np.uint8)))
             for _ in range(3)]
    layer = types.SimpleNamespace(gate=banks[0], up=banks[1], down=banks[2], router_w=None, router_bias=None)
    ids = torch.tensor([[0, 2], [2, 5], [0, 5]], dtype=torch.int32)            # experts 0, 2, 5 routed

    def csf_encode(sc):
        f, e, s = oracle.csf_encode(sc.numpy())
        return torch.from_numpy(f), torch.from_numpy(e.view(np.int32)), torch.from_numpy(s)

    def csf_decode(f, e, s, R_, C_, expert_offsets=None, out=None):
        full = torch.from_numpy(oracle.csf_decode(f.numpy(), e.numpy().view(np.uint32), s.numpy(), R_, C_))
        o = None if expert_offsets is None else expert_offsets.numpy()
        for ee in range(f.shape[0]):
            if o is None or o[ee + 1] > o[ee]:
                out[ee].copy_(full[ee])
        return out

    def permute(ids_, E_, ws):
        off, rs, sr = oracle.permute(ids_.numpy(), E_)
        return torch.from_numpy(off), torch.from_numpy(rs), torch.from_numpy(sr)

    fake = types.SimpleNamespace(csf_encode=csf_encode, csf_decode=csf_decode, permute=permute,
                                 route_topk=lambda *a: (ids, None), workspace=lambda *a: None)
    monkeypatch.setattr(bench, "time_calls", lambda fn, steps, *a, **kw: [fn() or 1.0 for _ in range(steps)])
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: None)
    res = bench.measure_csf(fake, wl, None, layer, 2, None, None, None, {"hbm_gbs": 1000.0}, "test")
    assert res["exact"] and res["experts_routed"] == 3
    want_all, want_routed = 0, 0
    for b in banks:
        f, e, s = oracle.csf_encode(b.scales.numpy())
        n_exc = np.diff(s)
        per = [f[x].nbytes + 4 * int(n_exc[x]) + 16 + R * C for x in range(E)]
        want_all += sum(per)
        want_routed += per[0] + per[2] + per[5]
    assert res["all_experts"]["algorithmic_bytes"] == want_all
    assert res["routed_experts"]["algorithmic_bytes"] == want_routed
    # 1 ms per call: achieved GB/s is bytes / 1e6
    assert res["all_experts"]["achieved"] == round(want_all / 1e6, 1)
