"""Benchmark: the 4-bit routed-expert MoE layer of Step-5-Preview on B200.

One step = one pass of the whole layer (router, bucketing, grouped gate/up +
SwiGLU, grouped down with routing weights, BF16 shared expert, combine) over
one batch of synthetic tokens, through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl reference]

Default workload: decode-shaped layer, int4 g128 W4A16, T = 8 tokens, hidden
4096, 352 experts of width 1536, top-8, BF16 shared expert.  Weights are bf16
N(0, 0.02^2) drawn on the GPU and converted by the library's quantiser;
activations bf16 N(0, 1); router fp32 N(0, 1/4096).  L2 is flushed (256 MB
write) before every timed step; each step is timed with CUDA events on the
launching stream and the flush is outside the events.

Under torchrun every rank runs an independent replica on its own GPU (the
layer has no cross-GPU exchange on this path); the step time is the maximum
over ranks and `value` sums all ranks' tokens.
"""
import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from weight_only_bit_route_b200 import synthetic as syn  # noqa: E402

METRIC = "MoE-layer tokens/s on 1 B200; % of HBM peak (decode) / BF16 tensor peak (prefill)"
UNIT = "tokens/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def describe(wl):
    return (f"{wl.name}: T={wl.T}, H={wl.H}, E={wl.E}, F={wl.F}, top-{wl.k}, "
            f"{'int4 g128' if wl.fmt == 'int4' else 'NVFP4'} W4A16 experts"
            f"{' + BF16 shared expert' if wl.shared else ''}{', Zipf-skewed routing' if wl.skew else ''}")


# ---------------------------------------------------------------------------
# bytes / FLOPs of the algorithm (not of the implementation)
# ---------------------------------------------------------------------------

def expert_bytes(wl):
    """Packed weights + scales (+ globals) of one routed expert, all three projections."""
    n = 3 * wl.F * wl.H
    if wl.fmt == "int4":
        return n // 2 + (n // 128) * 2
    return n // 2 + n // 16 + 3 * 4


def gateup_bytes_per_expert(wl):
    n = 2 * wl.F * wl.H
    if wl.fmt == "int4":
        return n // 2 + (n // 128) * 2
    return n // 2 + n // 16 + 2 * 4


def layer_bytes(wl, touched):
    shared = 3 * wl.F * wl.H * 2 if wl.shared else 0
    router = wl.E * wl.H * 4
    xy = 2 * wl.T * wl.H * 2
    return touched * expert_bytes(wl) + shared + router + xy


def layer_flops(wl):
    per_tok = wl.k * 2 * 3 * wl.F * wl.H + (2 * 3 * wl.F * wl.H if wl.shared else 0) + 2 * wl.E * wl.H
    return wl.T * per_tok


# ---------------------------------------------------------------------------
# building the layer on the GPU
# ---------------------------------------------------------------------------

def build_layer(moe, wl, seed=0, device="cuda"):
    x = torch.from_numpy(syn.gen_x(wl, seed).view(np.int16)).to(device).view(torch.bfloat16)
    Wr = torch.from_numpy(syn.gen_router(wl, seed)).to(device)
    b = syn.gen_bias(wl, seed)
    bias = None if b is None else torch.from_numpy(b).to(device)
    qws = torch.zeros(256, dtype=torch.uint8, device=device)
    banks = []
    for pi, which in enumerate(("gate", "up", "down")):
        out, inn = (wl.H, wl.F) if which == "down" else (wl.F, wl.H)
        if wl.fmt == "int4":
            packed = torch.empty(wl.E, out, inn // 8, dtype=torch.int32, device=device)
            scales = torch.empty(wl.E, out, inn // 128, dtype=torch.bfloat16, device=device)
            glob = None
        else:
            packed = torch.empty(wl.E, out, inn // 2, dtype=torch.uint8, device=device)
            scales = torch.empty(wl.E, out, inn // 16, dtype=torch.uint8, device=device)
            glob = torch.empty(wl.E, dtype=torch.float32, device=device)
        g = torch.Generator(device=device)
        for e in range(wl.E):
            g.manual_seed(seed * 7919 + pi * 104729 + e)
            w = (torch.randn(out, inn, generator=g, device=device, dtype=torch.float32) * wl.w_std).to(torch.bfloat16)
            if wl.fmt == "int4":
                p, s = moe.quantize_int4_g128(w)
                packed[e].copy_(p)
                scales[e].copy_(s)
            else:
                p, s, gl = moe.quantize_nvfp4(w, qws)
                packed[e].copy_(p)
                scales[e].copy_(s)
                glob[e:e + 1].copy_(gl)
        fmt = moe.FMT_INT4_G128 if wl.fmt == "int4" else moe.FMT_NVFP4
        banks.append(moe.Bank(fmt, packed, scales, glob))
    shared = None
    if wl.shared:
        shared = tuple(moe.Bank(moe.FMT_BF16, torch.from_numpy(syn.gen_shared(wl, w, seed).view(np.int16))
                                .to(device).view(torch.bfloat16)[None]) for w in ("gate", "up", "down"))
    layer = moe.MoELayer(*banks, router_w=Wr, top_k=wl.k, router_bias=bias, shared=shared)
    return x, layer


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML in a
    background thread while the timed region runs (read-only queries)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index, period_s=0.01):
        self.gpu, self.period = gpu_index, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None

    def _run(self):
        import pynvml
        h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        while not self.stop.is_set():
            self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
            try:
                r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
            except Exception:
                r = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
            for name, bit in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
            self.stop.wait(self.period)

    def __enter__(self):
        import threading
        self.stop = threading.Event()
        self.thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                self.gpu = int(vis.split(",")[self.gpu])
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        except Exception as e:   # no NVML: report no samples
            self.error = str(e)
        return self

    def __exit__(self, *a):
        self.stop.set()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# CPU baseline: the oracle on the host cores
# ---------------------------------------------------------------------------

def cpu_baseline(wl, moe, x, layer, budget_s=20.0):
    """Time the oracle's layer forward (router -> combine) on a bounded sample
    of the same workload's tokens (the layer is per-token)."""
    import oracle
    xb = x.view(torch.int16).cpu().numpy().view(np.uint16)
    Wr = layer.router_w.cpu().numpy()
    bias = None if layer.router_bias is None else layer.router_bias.cpu().numpy()

    def host_bank(b, experts):
        if b.fmt == moe.FMT_INT4_G128:
            packed = np.zeros(tuple(b.packed.shape), np.int32)
            scales = np.zeros(tuple(b.scales.shape), np.uint16)
            for e in experts:
                packed[e] = b.packed[e].cpu().numpy()
                scales[e] = b.scales[e].view(torch.int16).cpu().numpy().view(np.uint16)
            return oracle.Bank(oracle.FMT_INT4, packed, scales)
        packed = np.zeros(tuple(b.packed.shape), np.uint8)
        scales = np.zeros(tuple(b.scales.shape), np.uint8)
        for e in experts:
            packed[e] = b.packed[e].cpu().numpy()
            scales[e] = b.scales[e].cpu().numpy()
        return oracle.Bank(oracle.FMT_NVFP4, packed, scales, b.global_scale.cpu().numpy())

    T = x.shape[0]
    n = T
    t_route0 = time.perf_counter()
    ids, w = oracle.route(xb[:1], Wr, bias, wl.k)
    route_per_tok = time.perf_counter() - t_route0
    # estimate the per-token cost on one token, then size the sample to the budget
    experts = sorted(set(ids.ravel().tolist()))
    gate, up, down = (host_bank(b, experts) for b in (layer.gate, layer.up, layer.down))
    sh = None
    if layer.shared:
        sh = tuple(oracle.Bank(oracle.FMT_BF16, s.packed.view(torch.int16).cpu().numpy().view(np.uint16))
                   for s in layer.shared)
    t0 = time.perf_counter()
    oracle.moe_forward(xb[:1], ids, w, gate, up, down, shared=sh)
    per_tok = time.perf_counter() - t0 + route_per_tok
    n = int(max(1, min(T, budget_s / max(per_tok, 1e-9))))
    sample = xb[:n]
    ids, w = oracle.route(sample, Wr, bias, wl.k)
    experts = sorted(set(ids.ravel().tolist()))
    gate, up, down = (host_bank(b, experts) for b in (layer.gate, layer.up, layer.down))
    passes, done = 0, 0
    t0 = time.perf_counter()
    while True:
        ids, w = oracle.route(sample, Wr, bias, wl.k)
        oracle.moe_forward(sample, ids, w, gate, up, down, shared=sh)
        passes += 1
        done += n
        dt = time.perf_counter() - t0
        if dt >= min(10.0, budget_s):
            break
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return {"value": round(done / dt, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"first {n} of the workload's {T} tokens, router -> combine (oracle fp64 layer, "
                      f"OpenMP on {cores} threads), {passes} passes, {dt:.2f} s"}


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = syn.WORKLOADS[args.config]

    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from weight_only_bit_route_b200 import moe

    x, layer = build_layer(moe, wl)
    T = wl.T
    ws = moe.workspace(T, wl.H, wl.E, wl.F, wl.k)
    y = torch.empty_like(x)
    entry = moe.layer_decode if T <= 64 else moe.layer_forward
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        entry(x, layer, ws, out=y)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    status = moe.read_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")

    # routing facts for the algorithmic byte count
    ids, _ = moe.route_topk(x, layer.router_w, layer.router_bias, wl.k, ws)
    touched = int(torch.unique(ids).numel())

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = moe.launch_count()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
    launches = moe.launch_count() - launches0      # the library's own kernels in the timed region
    if dist:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms = float(np.mean(step_ms))
    if dist:
        t = torch.tensor([ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    value = world * T / (ms * 1e-3)

    # dominant kernel: grouped gate/up (+SwiGLU) through its own C-ABI call
    off, rs, sr = moe.permute(ids, wl.E, ws)
    R = T * wl.k
    h = torch.empty(R, wl.F, dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        moe.grouped_swiglu(x, off, rs, wl.k, layer.gate, layer.up, R, ws, out=h)
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        kev[i][0].record(stream)
        moe.grouped_swiglu(x, off, rs, wl.k, layer.gate, layer.up, R, ws, out=h)
        kev[i][1].record(stream)
    torch.cuda.synchronize()
    k_ms = float(np.mean([a.elapsed_time(b) for a, b in kev]))
    pk, pk_kind = peaks()
    # DRAM bytes (read + write) of one gate/up tcgen05_grouped_gemm launch, from the ncu captures summarised
    # under profiles/ for the current kernel; workloads without a capture report null
    traffic = {"decode_int4_T8": 395251456, "prefill_int4_T2048": 2472866648}.get(wl.name)
    decode = T <= 64
    if decode:
        kbytes = touched * gateup_bytes_per_expert(wl) + T * wl.H * 2
        achieved = kbytes / (k_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": traffic,
                "kernel": "tc_grouped_gemm gate/up+SwiGLU (with its activation gather)", "algorithmic_bytes": kbytes,
                "kernel_ms": round(k_ms, 5), "peak_source": f"{pk_kind} hbm_gbs"}
    else:
        kflops = 2 * 2 * wl.F * wl.H * R
        achieved = kflops / (k_ms * 1e-3) / 1e12
        peak = pk["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "kernel": "tc_grouped_gemm gate/up+SwiGLU (with its activation gather)",
                "algorithmic_flops": kflops, "kernel_ms": round(k_ms, 5), "peak_source": f"{pk_kind} bf16_tflops"}

    # end to end through the public API with host buffers
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    xd = torch.empty_like(x)
    eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps + 3):
        flush.zero_()
        j = i - 3
        if j >= 0:
            eev[j][0].record(stream)
        xd.copy_(xh, non_blocking=True)
        entry(xd, layer, ws, out=y)
        yh.copy_(y, non_blocking=True)
        if j >= 0:
            eev[j][1].record(stream)
    torch.cuda.synchronize()
    e_ms = float(np.mean([a.elapsed_time(b) for a, b in eev]))
    if dist:
        t = torch.tensor([e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e_ms = float(t.item())

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int4/e2m1 weights, bf16 activations, fp32 accumulate",
        "data": "synthetic (seeded; bf16 N(0,0.02^2) weights quantised by the library)",
        "config": {"workload": describe(wl), "T": T, "H": wl.H, "E": wl.E, "F": wl.F, "top_k": wl.k,
                   "format": wl.fmt, "shared_expert": wl.shared, "touched_experts": touched,
                   "l2": "flushed before every step (256 MB write, outside the events)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "algorithmic_bytes_per_step": layer_bytes(wl, touched),
                   "algorithmic_flops_per_step": layer_flops(wl),
                   "hbm_frac_whole_layer": round(layer_bytes(wl, touched) / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4)},
        "roofline": roof,
        "e2e": {"value": round(world * T / (e_ms * 1e-3), 1), "unit": UNIT,
                "h2d_bytes_per_step": int(x.numel() * 2), "d2h_bytes_per_step": int(y.numel() * 2)},
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, moe, x, layer)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args, wl, rank, world):
    """The oracle, as it stands, on the host cores (rank 0 only)."""
    if rank != 0:
        return
    import oracle
    x = syn.gen_x(wl)
    Wr = syn.gen_router(wl)
    bias = syn.gen_bias(wl)
    # each step: a bounded sample of the workload's tokens through router -> combine
    n = min(wl.T, 2)
    sample = x[:n]
    ids, w = oracle.route(sample, Wr, bias, wl.k)
    experts = sorted(set(ids.ravel().tolist()))

    class _W:
        pass
    fmt = oracle.FMT_INT4 if wl.fmt == "int4" else oracle.FMT_NVFP4
    banks = []
    for which in ("gate", "up", "down"):
        out, inn = (wl.H, wl.F) if which == "down" else (wl.F, wl.H)
        if wl.fmt == "int4":
            packed = np.zeros((wl.E, out, inn // 8), np.int32)
            scales = np.zeros((wl.E, out, inn // 128), np.uint16)
            glob = None
        else:
            packed = np.zeros((wl.E, out, inn // 2), np.uint8)
            scales = np.zeros((wl.E, out, inn // 16), np.uint8)
            glob = np.zeros(wl.E, np.float32)
        for e in experts:
            wb = syn.gen_expert(wl, which, e)
            if wl.fmt == "int4":
                packed[e], scales[e] = oracle.quant_int4_g128(wb)
            else:
                packed[e], scales[e], glob[e] = oracle.quant_nvfp4(wb)
        banks.append(oracle.Bank(fmt, packed, scales, glob))
    sh = None
    if wl.shared:
        sh = tuple(oracle.Bank(oracle.FMT_BF16, syn.gen_shared(wl, w)[None]) for w in ("gate", "up", "down"))
    for _ in range(args.warmup):
        pass   # the oracle has no warm-up state; skip untimed passes to bound the run time
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        ids, w = oracle.route(sample, Wr, bias, wl.k)
        oracle.moe_forward(sample, ids, w, *banks, shared=sh)
        times.append(time.perf_counter() - t0)
    ms = float(np.mean(times)) * 1e3
    value = n / (ms * 1e-3)
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    cb = {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
          "sample": f"{n} of the workload's {wl.T} tokens per step, router -> combine, OpenMP on {cores} threads"}
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp64 accumulate (oracle)", "data": "synthetic",
        "config": {"workload": describe(wl)}, "cpu_baseline": cb,
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


if __name__ == "__main__":
    main()
