"""Seeded synthetic inputs for the routed-expert MoE layer.

This module only draws random numbers: activations, router weights, the load
skew bias and bf16 expert weights, with the shapes and distributions of the
five workloads below.  It holds none of the layer's arithmetic (no quantiser,
no routing, no dequantisation), so both the CUDA path's tests and the CPU
oracle can take their inputs from it.

Streams: ``SeedSequence(seed).spawn(9)`` in the fixed order
``[x, router_w, bias_rank, gate, up, down, sh_gate, sh_up, sh_down]``; expert e
of a routed bank draws from ``spawn(E)[e]`` of its bank's stream, so any
single expert can be generated on its own.

bf16 values are returned as uint16 bit patterns (rounded from fp32 by torch's
round-to-nearest-even conversion).
"""
from dataclasses import dataclass

import numpy as np
import torch

STREAMS = ["x", "router_w", "bias_rank", "gate", "up", "down", "sh_gate", "sh_up", "sh_down"]


@dataclass(frozen=True)
class Workload:
    name: str
    T: int          # tokens
    H: int          # hidden size
    E: int          # routed experts
    F: int          # SwiGLU width of one expert
    k: int          # experts per token
    fmt: str        # "int4" (symmetric g128, bf16 scales) or "nvfp4"
    shared: bool    # one BF16 shared expert of width F
    router_std: float
    skew: bool      # per-expert additive logit bias giving a Zipf-like load
    w_std: float = 0.02
    skew_coef: float = 0.85


# Step-5-Preview's MoE layer: hidden 4096, a sigmoid router keeping 8 of 352
# routed experts, one shared expert, SwiGLU width 1536 (Step-5-Preview-Spark, At a
# glance; "Step 5 Preview: 92 narrow layers...", The shape).
WORKLOADS = {
    0: Workload("tiny_int4_T16_H1024_E32_F256", 16, 1024, 32, 256, 8, "int4", False,
                1.0 / np.sqrt(1024.0), False),
    1: Workload("decode_int4_T8", 8, 4096, 352, 1536, 8, "int4", True,
                1.0 / np.sqrt(4096.0), False),
    2: Workload("decode_nvfp4_T8", 8, 4096, 352, 1536, 8, "nvfp4", True,
                1.0 / np.sqrt(4096.0), False),
    3: Workload("prefill_int4_T2048", 2048, 4096, 352, 1536, 8, "int4", True,
                1.0 / np.sqrt(4096.0), False),
    4: Workload("prefill_nvfp4_T8192_zipf", 8192, 4096, 352, 1536, 8, "nvfp4", True,
                1.0 / np.sqrt(4096.0), True),
}


def _streams(seed):
    return dict(zip(STREAMS, np.random.SeedSequence(seed).spawn(len(STREAMS))))


def to_bf16_bits(a_f32):
    t = torch.from_numpy(np.ascontiguousarray(a_f32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def gen_x(wl: Workload, seed=0, T=None):
    """Activations bf16 N(0,1), [T, H] (uint16 bits)."""
    T = wl.T if T is None else T
    rng = np.random.Generator(np.random.PCG64(_streams(seed)["x"]))
    return to_bf16_bits(rng.standard_normal((T, wl.H), dtype=np.float32))


def gen_router(wl: Workload, seed=0):
    """Router weights fp32 N(0, router_std^2), [E, H]."""
    rng = np.random.Generator(np.random.PCG64(_streams(seed)["router_w"]))
    return (rng.standard_normal((wl.E, wl.H), dtype=np.float32) * np.float32(wl.router_std))


def gen_bias(wl: Workload, seed=0):
    """Per-expert logit bias b_e = -c * ln(rank_e), rank_e = 1 + a seeded
    permutation of 0..E-1 (skewed workloads only; None otherwise)."""
    if not wl.skew:
        return None
    rng = np.random.Generator(np.random.PCG64(_streams(seed)["bias_rank"]))
    rank = 1 + rng.permutation(wl.E)
    return (-wl.skew_coef * np.log(rank.astype(np.float64))).astype(np.float32)


def gen_expert(wl: Workload, which: str, e: int, seed=0):
    """bf16 N(0, w_std^2) weights of routed expert e in the pages' [out, in]
    orientation: gate/up [F, H], down [H, F]."""
    assert which in ("gate", "up", "down")
    ss = _streams(seed)[which].spawn(wl.E)[e]
    rng = np.random.Generator(np.random.PCG64(ss))
    shape = (wl.H, wl.F) if which == "down" else (wl.F, wl.H)
    return to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(wl.w_std))


def gen_shared(wl: Workload, which: str, seed=0):
    """bf16 N(0, w_std^2) shared-expert weights: gate/up [F, H], down [H, F]."""
    assert which in ("gate", "up", "down")
    rng = np.random.Generator(np.random.PCG64(_streams(seed)["sh_" + which]))
    shape = (wl.H, wl.F) if which == "down" else (wl.F, wl.H)
    return to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(wl.w_std))


def gen_random_codes(wl: Workload, which: str, e: int, seed=0):
    """Uniformly random packed codes and plausible scales for routed expert e,
    as raw storage (no quantiser involved).  Used where a full-size bank is
    needed but only some experts are checked against the oracle.

    int4:  packed int32 [out, in/8] (any 32-bit pattern), scales bf16 bits
           [out, in/128] with values |N(0, (w_std/4)^2)| rounded to bf16.
    nvfp4: packed uint8 [out, in/2], scales uint8 E4M3 bytes in [0x28, 0x70]
           (0.5 .. 256), global fp32 = w_std / 448.
    """
    ss = _streams(seed + 1_000_003)[which].spawn(wl.E)[e]
    rng = np.random.Generator(np.random.PCG64(ss))
    out, inn = (wl.H, wl.F) if which == "down" else (wl.F, wl.H)
    if wl.fmt == "int4":
        packed = rng.integers(0, 2**32, size=(out, inn // 8), dtype=np.uint64).astype(np.uint32).view(np.int32)
        sc = np.abs(rng.standard_normal((out, inn // 128), dtype=np.float32)) * np.float32(wl.w_std / 4)
        return packed, to_bf16_bits(sc), None
    packed = rng.integers(0, 256, size=(out, inn // 2), dtype=np.uint8)
    sc = rng.integers(0x28, 0x71, size=(out, inn // 16), dtype=np.uint8)
    return packed, sc, np.float32(wl.w_std / 448.0)
