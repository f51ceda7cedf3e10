"""Benchmark: the 4-bit routed-expert MoE layer of Step-5-Preview on B200.

One step = one pass of the whole layer (router, bucketing, grouped gate/up +
SwiGLU, grouped down with routing weights, BF16 shared expert, combine) over
one batch of synthetic tokens, through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--per-config 2,3,4]
                    [--impl reference]

Headline workload (the line's value): decode-shaped layer, int4 g128 W4A16,
T = 8 tokens, hidden 4096, 352 experts of width 1536, top-8, BF16 shared
expert.  The other workloads (NVFP4 decode, int4 prefill T = 2048, NVFP4
prefill T = 8192 with Zipf-skewed routing) go into `per_config` on the same
line, each with its layer time (mean, median, p10, p90), its dominant-kernel
roofline, its whole-layer roofline and the time of each step through its own
C-ABI call; the NVFP4 decode workload also carries the CSF expansion of its
layer's scales (`csf`).  With one process, `expert_parallel` times the same
layer split by experts over a one-rank NCCL group.  Weights are bf16
N(0, 0.02^2) drawn on the GPU and converted by
the library's quantisers; activations bf16 N(0, 1); router fp32 N(0, 1/4096).
L2 is flushed (256 MB write) before every timed call; each call is timed with
CUDA events on the launching stream and the flush is outside the events.

Under torchrun every rank runs an independent replica on its own GPU (the
layer has no cross-GPU exchange on this path); the step time is the maximum
over ranks and `value` sums all ranks' tokens.
"""
import argparse
import json
import os
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from weight_only_bit_route_b200 import synthetic as syn  # noqa: E402

METRIC = "MoE-layer tokens/s on 1 B200; % of HBM peak (decode) / BF16 tensor peak (prefill)"
UNIT = "tokens/s"
W4A4_IN_GATEUP = 4.5 / 2688.0       # activation global scales of the W4A4 runs (amax / (6 * 448))
W4A4_IN_DOWN = 8.0 / 2688.0
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
    """Samples SM clock and clock-event reasons through NVML (read-only
    queries): a background thread every `period_s` while the sampler is open,
    plus a synchronous sample whenever mark() is called (before and after
    every timed loop), so that short timed regions still get samples."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index, period_s=0.005):
        self.gpu, self.period = gpu_index, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.handle = None
        self.error = None

    def _sample(self):
        import pynvml
        self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(self.handle, pynvml.NVML_CLOCK_SM)))
        try:
            r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
        except Exception:
            r = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
        for name, bit in self.REASONS.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        while not self.stop.is_set():
            self._sample()
            self.stop.wait(self.period)

    def mark(self):
        if self.handle is not None:
            self._sample()

    def __enter__(self):
        import threading
        self.stop = threading.Event()
        self.thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            gpu = self.gpu
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                gpu = int(vis.split(",")[self.gpu])
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(gpu)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        except Exception as e:   # no NVML: report no samples
            self.error = str(e)
            self.handle = None
        return self

    def __exit__(self, *a):
        self.stop.set()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "error": self.error}
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
                      f"OpenMP on {cores} threads), {passes} passes, {dt:.2f} s",
            "single_thread": oracle_single_thread(oracle, sample[:1], Wr, bias, wl.k, (gate, up, down), sh,
                                                  min(8.0, budget_s / 2)),
            "host_threads": os.cpu_count()}


def oracle_single_thread(oracle, sample, Wr, bias, k, banks, sh, budget_s):
    """The oracle's layer forward on one OpenMP thread: passes over a one-token sample until budget_s has gone."""
    oracle.set_threads(1)
    try:
        passes = 0
        t0 = time.perf_counter()
        while True:
            ids, w = oracle.route(sample, Wr, bias, k)
            oracle.moe_forward(sample, ids, w, *banks, shared=sh)
            passes += 1
            dt = time.perf_counter() - t0
            if dt >= budget_s:
                break
    finally:
        oracle.set_threads(0)
    return {"value": round(passes * sample.shape[0] / dt, 3), "unit": UNIT, "cores": 1,
            "sample": f"{sample.shape[0]} token, router -> combine on one thread, {passes} passes, {dt:.2f} s"}


# ---------------------------------------------------------------------------
# measurement
# ---------------------------------------------------------------------------

# DRAM bytes (read + write) of one launch of the dominant kernel, from the launch lists of the bench's own
# command with `--metrics gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum` (summarised under
# profiles/), keyed by workload and by the hash of the GEMM's code (comments aside) at the time of the capture:
# a figure whose kernel has changed since is reported as null.
TRAFFIC = {
    ("decode_int4_T8", "94e237ba6c42a308"): 390216960 + 591616,
    ("decode_nvfp4_T8", "94e237ba6c42a308"): 425606912 + 201216,
}


def gemm_source_hash():
    """Hash of the GEMM's code with comments and blank space removed (a comment edit keeps the kernel)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in ("gemm_tc.cu", "tc_ptx.cuh", "moe_internal.cuh"):
        src = open(os.path.join(ROOT, "weight_only_bit_route_b200", "csrc", f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update(re.sub(r"\s+", "", src).encode())
    return h.hexdigest()[:16]


def oracle_free_f16(wl, seed=0):
    """The workload's activations drawn in fp32 and rounded to fp16 (not through bf16)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed).spawn(9)[0]))
    return rng.standard_normal((wl.T, wl.H), dtype=np.float32).astype(np.float16)


def _pcts(ms):
    a = np.asarray(ms, np.float64)
    return {"mean": round(float(a.mean()), 5), "median": round(float(np.median(a)), 5),
            "p10": round(float(np.percentile(a, 10)), 5), "p90": round(float(np.percentile(a, 90)), 5)}


def time_calls(fn, steps, flush, stream, clk, warmup=3):
    """CUDA-event times (ms) of `steps` calls of fn on `stream`, L2 flushed
    before each call outside the events."""
    for _ in range(warmup):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    clk.mark()
    for i in range(steps):
        flush.zero_()
        evs[i][0].record(stream)
        fn()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    clk.mark()
    return [a.elapsed_time(b) for a, b in evs]


def step_times(moe, wl, x, layer, ws, steps, flush, stream, clk):
    """Median time of each step through its own C-ABI call (a1..a6)."""
    T, k = x.shape[0], wl.k
    R = T * k
    ids, tw = moe.route_topk(x, layer.router_w, layer.router_bias, k, ws)
    off, rs, sr = moe.permute(ids, wl.E, ws)
    h = torch.empty(R, wl.F, dtype=torch.bfloat16, device="cuda")
    yp = torch.empty(R, wl.H, dtype=torch.bfloat16, device="cuda")
    y = torch.empty_like(x)
    out = {}
    med = lambda v: round(float(np.median(v)), 5)
    out["a1_router"] = med(time_calls(lambda: moe.route_topk(x, layer.router_w, layer.router_bias, k, ws),
                                      steps, flush, stream, clk))
    out["a2_bucketing"] = med(time_calls(lambda: moe.permute(ids, wl.E, ws), steps, flush, stream, clk))
    out["a3_gateup_swiglu"] = med(time_calls(
        lambda: moe.grouped_swiglu(x, off, rs, k, layer.gate, layer.up, R, ws, out=h), steps, flush, stream, clk))
    out["a4_down"] = med(time_calls(lambda: moe.grouped_down(h, off, rs, tw.view(-1), layer.down, ws, out=yp),
                                    steps, flush, stream, clk))
    ys = None
    if layer.shared:
        so = torch.tensor([0, T], dtype=torch.int32, device="cuda")
        srs = torch.arange(T, dtype=torch.int32, device="cuda") * k
        hs = torch.empty(T, wl.F, dtype=torch.bfloat16, device="cuda")
        ys = torch.empty_like(x)

        def shared():
            moe.grouped_swiglu(x, so, srs, k, layer.shared[0], layer.shared[1], T, ws, out=hs)
            moe.grouped_down(hs, so, srs, None, layer.shared[2], ws, out=ys)
        out["a5_shared_expert"] = med(time_calls(shared, steps, flush, stream, clk))
    out["a6_combine"] = med(time_calls(lambda: moe.unpermute_combine(yp, sr, T, k, ys, out=y),
                                       steps, flush, stream, clk))
    return out


def measure(moe, wl, x, layer, args, flush, stream, clk, pk, pk_kind, per_step=True, fp4=False):
    """Layer timing (+ dominant-kernel roofline and per-step times) of one workload."""
    T = wl.T
    ws = moe.workspace(T, wl.H, wl.E, wl.F, wl.k)
    y = torch.empty_like(x)
    entry = moe.layer_decode if T <= 64 else moe.layer_forward
    step = lambda: entry(x, layer, ws, out=y)
    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    status = moe.read_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")
    # the step-level calls take bf16 activations: an fp16 layer's routing facts and dominant-kernel
    # time come from the same values rounded to bf16
    xb = x if x.dtype == torch.bfloat16 else x.to(torch.bfloat16)
    ids, _ = moe.route_topk(xb, layer.router_w, layer.router_bias, wl.k, ws)
    touched = int(torch.unique(ids).numel())
    torch.cuda.synchronize()
    launches0 = moe.launch_count()
    eager_list = time_calls(step, args.steps, flush, stream, clk, warmup=0)
    eager_launches = moe.launch_count() - launches0
    # the same call recorded once as a CUDA graph (moe_layer_graph_*) and replayed: the layer's
    # kernels without the host's per-call launch work
    graph = moe.LayerGraph(x, layer, ws, out=y)
    for _ in range(3):
        flush.zero_()
        graph.launch()
    torch.cuda.synchronize()
    launches0 = moe.launch_count()
    ms_list = time_calls(graph.launch, args.steps, flush, stream, clk, warmup=0)
    launches = moe.launch_count() - launches0
    # dominant kernel: grouped gate/up (+ SwiGLU) through its own C-ABI call
    off, rs, sr = moe.permute(ids, wl.E, ws)
    R = T * wl.k
    h = torch.empty(R, wl.F, dtype=torch.bfloat16, device="cuda")
    k_ms = float(np.mean(time_calls(lambda: moe.grouped_swiglu(xb, off, rs, wl.k, layer.gate, layer.up, R, ws, out=h),
                                    args.steps, flush, stream, clk)))
    if moe.read_status(ws) != 0:
        raise RuntimeError("device status set during timing")
    ms = float(np.mean(ms_list))
    decode = T <= 64
    traffic = None if fp4 else TRAFFIC.get((wl.name, gemm_source_hash()))    # (W4A4 runs another kernel)
    lbytes, lflops = layer_bytes(wl, touched), layer_flops(wl)
    kernel_name = "tc_grouped_gemm gate/up+SwiGLU (with its activation pre-pass)"
    if decode:
        kbytes = touched * gateup_bytes_per_expert(wl) + T * wl.H * 2
        achieved = kbytes / (k_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": traffic, "kernel": kernel_name,
                "algorithmic_bytes": kbytes, "kernel_ms": round(k_ms, 5), "peak_source": f"{pk_kind} hbm_gbs"}
        layer_roof = {"bound": "hbm", "algorithmic_bytes": lbytes,
                      "achieved_gbs": round(lbytes / (ms * 1e-3) / 1e9, 1),
                      "frac": round(lbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
    else:
        kflops = 2 * 2 * wl.F * wl.H * R
        achieved = kflops / (k_ms * 1e-3) / 1e12
        # W4A4 runs on the FP4 tensor cores: its peak is the measured BF16 one times the nominal
        # dense ratio FP4 / BF16 (9 / 2.25 PFLOP/s)
        kpeak = pk["bf16_tflops"] * (4.0 if fp4 else 1.0)
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(kpeak, 1), "unit": "TFLOP/s",
                "frac": round(achieved / kpeak, 4), "traffic": traffic, "kernel": kernel_name,
                "algorithmic_flops": kflops, "kernel_ms": round(k_ms, 5),
                "peak_source": f"{pk_kind} bf16_tflops" + (" x 4 (FP4 / BF16 nominal dense ratio)" if fp4 else "")}
        tf = lflops / (ms * 1e-3) / 1e12
        layer_roof = {"bound": "tensor", "algorithmic_flops": lflops, "achieved_tflops": round(tf, 1),
                      "frac_burst": round(tf / pk["bf16_tflops"], 4),
                      "frac_sustained": round(tf / pk.get("bf16_tflops_sustained", pk["bf16_tflops"]), 4),
                      "algorithmic_bytes": lbytes,
                      "hbm_frac": round(lbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
    e_ms = float(np.mean(eager_list))
    res = {"workload": describe(wl), "T": T, "format": wl.fmt, "touched_experts": touched,
           "tokens_per_s": round(T / (ms * 1e-3), 1), "layer_ms": _pcts(ms_list),
           "roofline": roof, "layer_roofline": layer_roof, "gpu_launches_per_step": launches / args.steps,
           "eager": {"tokens_per_s": round(T / (e_ms * 1e-3), 1), "layer_ms": _pcts(eager_list),
                     "gpu_launches_per_step": eager_launches / args.steps}}
    if per_step:
        res["steps_ms"] = step_times(moe, wl, x, layer, ws, args.steps, flush, stream, clk)
    return res, ms, ms_list, touched, launches, ws, graph


def measure_csf(moe, wl, x, layer, steps, flush, stream, clk, pk, pk_kind):
    """CSF scale expansion ("Step-5-Preview-NVFP4-Local", Format and Size) of the layer's NVFP4 block scales,
    encoded once here: all experts of the three projections (one layer's scales before it runs) and only the
    experts this workload routes to.  HBM-bound: the algorithmic bytes are the planes read (fixed, the
    exceptions, starts) plus the scale bytes written, for the experts expanded."""
    banks = (layer.gate, layer.up, layer.down)
    planes = []
    for bank in banks:
        _, R, C = bank.scales.shape
        f, e, s = moe.csf_encode(bank.scales)
        planes.append((f, e, s, R, C, torch.empty_like(bank.scales)))
    ws = moe.workspace(wl.T, wl.H, wl.E, wl.F, wl.k)
    ids, _ = moe.route_topk(x, layer.router_w, layer.router_bias, wl.k, ws)
    off, _, _ = moe.permute(ids, wl.E, ws)

    def expand(offsets):
        for f, e, s, R, C, out in planes:
            moe.csf_decode(f, e, s, R, C, expert_offsets=offsets, out=out)

    expand(None)
    torch.cuda.synchronize()
    exact = all(torch.equal(p[5], b.scales) for p, b in zip(planes, banks))
    live = (off[1:] > off[:-1]).cpu().numpy()
    bytes_all, bytes_routed = 0, 0
    for f, e, s, R, C, out in planes:
        st = s.cpu().numpy()
        per_e = f[0].numel() + R * C + 16                      # fixed slab + scales written + starts pair
        exc_e = (st[1:] - st[:-1]) * 4
        bytes_all += int(f.shape[0] * per_e + exc_e.sum())
        bytes_routed += int(live.sum() * per_e + exc_e[live].sum())
    res = {"exact": bool(exact), "experts_routed": int(live.sum()), "kernel": "csf_expand + csf_patch, x3 projections",
           "peak": pk["hbm_gbs"], "unit": "GB/s", "peak_source": f"{pk_kind} hbm_gbs"}
    for name, offsets, nbytes in (("all_experts", None, bytes_all), ("routed_experts", off, bytes_routed)):
        ms = float(np.mean(time_calls(lambda: expand(offsets), steps, flush, stream, clk)))
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[name] = {"ms": round(ms, 5), "algorithmic_bytes": nbytes, "achieved": round(gbs, 1),
                     "frac": round(gbs / pk["hbm_gbs"], 4)}
    return res


def measure_ep_one_rank(moe, wl, x, layer, steps, flush, stream, clk, backend="nccl", ops=None):
    """The expert-parallel layer (weight_only_bit_route_b200/ep.py) as a one-rank NCCL group: every step in the
    library's kernels and the rows through NCCL's all-to-all, which on one rank is a local copy.  Its time
    against the fused layer's is the cost of the split's bookkeeping (the host reads of the split sizes, the
    exchanges, the per-rank grouping); its output must equal the fused layer's bit for bit.  backend and ops
    exist for a CPU test of this function (gloo, the oracle's steps)."""
    import datetime
    import socket

    import torch.distributed as dist

    from weight_only_bit_route_b200 import ep
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group(backend, rank=0, world_size=1, init_method=f"tcp://127.0.0.1:{port}",
                            timeout=datetime.timedelta(seconds=60))
    try:
        lay = ep.ExpertParallelMoE(layer.gate, layer.up, layer.down, layer.router_w, top_k=wl.k,
                                   router_bias=layer.router_bias, shared=layer.shared, max_tokens=wl.T, ops=ops)
        ws = moe.workspace(wl.T, wl.H, wl.E, wl.F, wl.k)
        y_ref = moe.layer_decode(x, layer, ws)
        y = lay.forward(x)
        torch.cuda.synchronize()
        exact = bool(torch.equal(y, y_ref))
        ms_list = time_calls(lambda: lay.forward(x), steps, flush, stream, clk)
        torch.cuda.synchronize()
        return {"world": 1, "exact_vs_fused_layer": exact, "layer_ms": _pcts(ms_list),
                "tokens_per_s": round(wl.T / (float(np.mean(ms_list)) * 1e-3), 1),
                "note": "one rank: the all-to-all moves rows within this GPU; several GPUs are not measured"}
    finally:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=1, help="the headline workload")
    ap.add_argument("--per-config", default="2,3,4,2w,4w,1h",
                    help="other workloads measured into per_config (comma list; a trailing 'w' runs an NVFP4 "
                         "workload as W4A4, activations quantised on the fly; a trailing 'h' runs it with fp16 "
                         "activations; or 'none')")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = syn.WORKLOADS[args.config]
    others = [] if args.per_config == "none" else [c.strip() for c in args.per_config.split(",") if c.strip()]
    others = [c for c in others if c != str(args.config)]

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

    # weights: one int4 and one NVFP4 bank set (the workloads of a format share their weights)
    layers = {}

    def layer_for(w):
        if w.fmt not in layers:
            layers[w.fmt] = build_layer(moe, w)[1]
        lay = layers[w.fmt]
        b = syn.gen_bias(w)
        lay.router_bias = None if b is None else torch.from_numpy(b).cuda()
        return lay

    def x_for(w):
        return torch.from_numpy(syn.gen_x(w).view(np.int16)).cuda().view(torch.bfloat16)

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    pk, pk_kind = peaks()
    T = wl.T
    x = x_for(wl)
    layer = layer_for(wl)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        head, ms, ms_list, touched, launches, ws, graph = measure(moe, wl, x, layer, args, flush, stream, clk,
                                                                  pk, pk_kind)
        if dist:
            t = torch.tensor([ms], device="cuda")
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ms = float(t.item())
        value = world * T / (ms * 1e-3)

        # end to end through the public API with host buffers: each step copies its tokens into the
        # recorded layer's input, replays the layer and copies the output back
        xh = x.cpu().pin_memory()
        yh = torch.empty_like(xh).pin_memory()

        def e2e_step():
            graph.x.copy_(xh, non_blocking=True)
            graph.launch()
            yh.copy_(graph.y, non_blocking=True)
        e_ms = float(np.mean(time_calls(e2e_step, args.steps, flush, stream, clk)))
        if dist:
            t = torch.tensor([e_ms], device="cuda")
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())

        per_config = {}
        for c in others:
            w4a4 = c.endswith("w")
            f16 = c.endswith("h")
            w2 = syn.WORKLOADS[int(c.rstrip("wh"))]
            lay = layer_for(w2)
            x2 = x_for(w2)
            if f16:
                # fp16 activations: the same draw as fp16 values
                x2 = torch.from_numpy(oracle_free_f16(w2)).cuda()
                lay.act_f16 = True
            if w4a4:
                if w2.fmt != "nvfp4":
                    continue
                # static activation scales standing in for calibrated ones: the inputs' typical
                # amax / (6 * 448) (x ~ N(0, 1) over 4096 elements; h of these weights stays below ~8)
                lay.gate.input_scale = torch.full((w2.E,), W4A4_IN_GATEUP, dtype=torch.float32, device="cuda")
                lay.down.input_scale = torch.full((w2.E,), W4A4_IN_DOWN, dtype=torch.float32, device="cuda")
            try:
                res = measure(moe, w2, x2, lay, args, flush, stream, clk, pk, pk_kind, fp4=w4a4,
                              per_step=not f16)[0]
                if c == "2":
                    # the scales of this NVFP4 layer through the compressed scale format's expansion
                    try:
                        res["csf"] = measure_csf(moe, w2, x2, lay, args.steps, flush, stream, clk, pk, pk_kind)
                    except Exception as err:         # recorded, so that the rest of the line still prints
                        res["csf"] = {"error": f"{type(err).__name__}: {err}"[:300]}
            except Exception as err:                 # one workload's failure is recorded, not fatal to the line
                res = {"workload": describe(w2), "error": f"{type(err).__name__}: {err}"[:300]}
            if w4a4:
                res["workload"] += " (W4A4: NVFP4 activations, static input scales)"
                lay.gate.input_scale = lay.down.input_scale = None
            if f16:
                res["workload"] += " (fp16 activations)"
                lay.act_f16 = False
            per_config[c] = res
            torch.cuda.empty_cache()
        layer = layer_for(wl)          # restore the headline workload's bias for the CPU leg

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
                   "algorithmic_flops_per_step": layer_flops(wl)},
        "layer_ms": head["layer_ms"],
        "eager": head["eager"],
        "roofline": head["roofline"],
        "layer_roofline": head["layer_roofline"],
        "steps_ms": head.get("steps_ms"),
        "e2e": {"value": round(world * T / (e_ms * 1e-3), 1), "unit": UNIT,
                "h2d_bytes_per_step": int(x.numel() * 2), "d2h_bytes_per_step": int(x.numel() * 2)},
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "per_config": per_config,
    }
    if world == 1 and T <= 64:
        # the expert-parallel split of the same layer, on one rank (recorded, so that an error cannot drop the line)
        try:
            line["expert_parallel"] = measure_ep_one_rank(moe, wl, x, layer, min(args.steps, 50), flush, stream,
                                                          ClockSampler(local_rank))
        except Exception as err:
            line["expert_parallel"] = {"error": f"{type(err).__name__}: {err}"[:300]}
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
    for _ in range(args.warmup):                     # untimed passes of the same sample
        ids, w = oracle.route(sample, Wr, bias, wl.k)
        oracle.moe_forward(sample, ids, w, *banks, shared=sh)
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
          "sample": f"{n} of the workload's {wl.T} tokens per step, router -> combine, OpenMP on {cores} threads",
          "single_thread": oracle_single_thread(oracle, sample[:1], Wr, bias, wl.k, banks, sh, 5.0),
          "host_threads": os.cpu_count()}
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp64 accumulate (oracle)", "data": "synthetic",
        "config": {"workload": describe(wl)}, "cpu_baseline": cb,
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


if __name__ == "__main__":
    main()
