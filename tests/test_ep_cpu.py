"""Expert-parallel layer (weight_only_bit_route_b200/ep.py) on two and four CPU ranks over gloo.

Each rank owns an equal share of the routed experts and routes its own tokens; the steps run in the oracle (an injected
step set: the collectives and the bookkeeping around them are what is tested here, the steps' kernels are
tested on the GPU).  Bars: each rank's output is bit-identical to the same steps run on one process with every
expert local, and within the layer tolerance of the oracle's fp64 layer.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _from_bits(b):
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)


def _to_bf16(v):
    u = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7fff + ((u >> 16) & 1)) >> 16).astype(np.uint16)


class RefOps:
    """The layer's steps in the oracle, with the GPU path's roundings (h and the expert outputs to bf16)."""

    def __init__(self, oracle, P, e0, e1):
        self.o, self.P, self.k = oracle, P, P.wl.k
        self.e_local = e1 - e0
        sl = slice(e0, e1)
        self.banks = {w: oracle.Bank(b.fmt, b.packed[sl], b.scales[sl],
                                     None if b.global_scale is None else b.global_scale[sl])
                      for w, b in P.banks.items()}

    def route(self, x):
        ids, w = self.o.route(_bits(x), self.P.Wr, self.P.bias, self.k)
        return torch.from_numpy(ids), torch.from_numpy(w)

    def group(self, owner, world):
        off, rs, sr = self.o.permute(owner.numpy(), world)
        return torch.from_numpy(off), torch.from_numpy(rs), torch.from_numpy(sr)

    def experts(self, xr, er, wr):
        R = xr.shape[0]
        if R == 0:
            return torch.empty_like(xr)
        off, rs, sr = self.o.permute(er.numpy().reshape(R, 1), self.e_local)
        rows = np.arange(R, dtype=np.int32)
        h = self.o.grouped_swiglu(_bits(xr), off, rs, 1, self.banks["gate"], self.banks["up"], rows)
        yp = _to_bf16(self.o.grouped_down(_to_bf16(h), off, rs, wr.numpy(), self.banks["down"], rows))
        return _from_bits(yp[sr])

    def shared_expert(self, x):
        if self.P.shared is None:
            return None
        T = x.shape[0]
        so = np.array([0, T], np.int32)
        srs = (np.arange(T) * self.k).astype(np.int32)
        rows = np.arange(T, dtype=np.int32)
        hs = self.o.grouped_swiglu(_bits(x), so, srs, self.k, self.P.shared[0], self.P.shared[1], rows)
        return _from_bits(_to_bf16(self.o.grouped_down(_to_bf16(hs), so, srs, None, self.P.shared[2], rows)))

    def combine(self, y_back, slot_pos, T, shared_out):
        sh = None if shared_out is None else _bits(shared_out)
        return _from_bits(_to_bf16(self.o.combine(_bits(y_back), slot_pos.numpy(), T, self.k, sh)))


def _worker(rank, world, counts, port, results):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path[:0] = [root, os.path.join(root, "tests")]
    import torch.distributed as dist
    import oracle
    from problems import build, layer_tolerance
    from weight_only_bit_route_b200 import ep
    from weight_only_bit_route_b200 import synthetic as syn

    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}")
    try:
        wl = syn.WORKLOADS[0]
        P = build(0, "random", experts=list(range(wl.E)), shared=True)
        x = _from_bits(syn.gen_x(wl, seed=100 + rank, T=counts[rank]))
        e_per = wl.E // world
        ops = RefOps(oracle, P, rank * e_per, (rank + 1) * e_per)
        layer = ep.ExpertParallelMoE(ops.banks["gate"], ops.banks["up"], ops.banks["down"], P.Wr, top_k=wl.k,
                                     max_tokens=16, ops=ops)
        y = _bits(layer.forward(x))
        # the same steps on one process, every expert local
        full = RefOps(oracle, P, 0, wl.E)
        ids, w = full.route(x)
        T = x.shape[0]
        assert y.shape == (T, wl.H)
        off, rs, sr = full.group(torch.zeros(T, wl.k, dtype=torch.int32), 1)
        ys = full.experts(x.index_select(0, rs.to(torch.int64) // wl.k), ids.view(-1)[rs.to(torch.int64)],
                          w.view(-1)[rs.to(torch.int64)])
        y1 = _bits(full.combine(ys, sr, T, full.shared_expert(x)))
        ref = oracle.moe_forward(_bits(x), ids.numpy(), w.numpy(), P.banks["gate"], P.banks["up"], P.banks["down"],
                                 shared=P.shared)
        got = oracle.bf16_to_f32(y).astype(np.float64)
        ok_tol = T == 0 or bool(np.all(np.abs(got - ref) <= layer_tolerance(ref)))
        results.put((rank, bool(np.array_equal(y, y1)), ok_tol, int(T)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("counts", [(16, 13), (16, 13, 0, 5)], ids=["two_ranks_ragged", "four_ranks_one_empty"])
def test_expert_parallel_gloo(counts):
    """Ragged token counts; on four ranks one rank has no tokens and still takes part in every exchange."""
    world = len(counts)
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, counts, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0] * world, f"rank exit codes {codes}"
    got = sorted(results.get(timeout=5) for _ in range(world))
    assert [g[3] for g in got] == list(counts)
    for rank, same, within, _ in got:
        assert same, f"rank {rank}: the expert-parallel result differs from the one-process composition"
        assert within, f"rank {rank}: outside the layer tolerance of the oracle"


def _refusal_worker(rank, world, port, results):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path[:0] = [root, os.path.join(root, "tests")]
    import torch.distributed as dist
    import oracle
    from problems import build
    from weight_only_bit_route_b200 import ep
    from weight_only_bit_route_b200 import synthetic as syn

    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}",
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = syn.WORKLOADS[0]
        P = build(0, "random", experts=list(range(wl.E)), shared=False)
        e_per = wl.E // world
        ops = RefOps(oracle, P, rank * e_per, (rank + 1) * e_per)
        layer = ep.ExpertParallelMoE(ops.banks["gate"], ops.banks["up"], ops.banks["down"], P.Wr, top_k=wl.k,
                                     max_tokens=8, ops=ops)
        # rank 1's batch is one token too many: both ranks must raise, neither may wait for the other
        x = _from_bits(syn.gen_x(wl, seed=200 + rank, T=9 if rank == 1 else 4))
        try:
            layer.forward(x)
            raised = ""
        except ValueError as e:
            raised = str(e)
        # the group is still in step: a valid call afterwards completes on both ranks
        y = layer.forward(x[:3].contiguous())
        results.put((rank, raised, tuple(y.shape)))
    finally:
        dist.destroy_process_group()


def test_expert_parallel_refusal_reaches_every_rank():
    """A batch above max_tokens on one rank makes every rank raise ValueError after the counts' exchange (no rank
    is left in a collective), and the next call runs normally."""
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_refusal_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], f"rank exit codes {codes}"
    got = sorted(results.get(timeout=5) for _ in range(2))
    assert "refused" in got[0][1], got[0]
    assert "exceeds max_tokens" in got[1][1], got[1]
    assert [g[2] for g in got] == [(3, 1024), (3, 1024)]


def _leaver_worker(rank, world, port, results):
    import sys
    import time
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path[:0] = [root, os.path.join(root, "tests")]
    import torch.distributed as dist
    import oracle
    from problems import build
    from weight_only_bit_route_b200 import ep
    from weight_only_bit_route_b200 import synthetic as syn

    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}",
                            timeout=datetime.timedelta(seconds=10))
    if rank == 1:
        # this rank leaves between calls, with nothing in flight
        dist.destroy_process_group()
        return
    wl = syn.WORKLOADS[0]
    P = build(0, "random", experts=list(range(wl.E)), shared=False)
    e_per = wl.E // world
    ops = RefOps(oracle, P, 0, e_per)
    layer = ep.ExpertParallelMoE(ops.banks["gate"], ops.banks["up"], ops.banks["down"], P.Wr, top_k=wl.k,
                                 max_tokens=8, ops=ops)
    t0 = time.monotonic()
    try:
        layer.forward(_from_bits(syn.gen_x(wl, seed=300, T=4)))
        err = ""
    except Exception as e:                  # the backend's error type differs between versions
        err = type(e).__name__
    results.put((rank, err, time.monotonic() - t0))


def test_expert_parallel_rank_that_left():
    """A rank that leaves the group between calls: the other rank's next call ends with an error from its first
    collective, within the group's timeout, instead of waiting for ever."""
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_leaver_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], f"rank exit codes {codes}"
    rank, err, secs = results.get(timeout=5)
    assert rank == 0 and err, "the remaining rank's call did not fail"
    assert err != "ValueError", "the call failed before its first collective"
    assert secs < 60


def test_expert_parallel_argument_checks():
    """Experts that do not split evenly over the ranks, and batches above max_tokens, are refused."""
    import torch.distributed as dist
    from weight_only_bit_route_b200 import ep

    class _Bank:
        def __init__(self, E):
            self.E = E

    class _Ops:
        pass

    dist.init_process_group("gloo", rank=0, world_size=1, init_method=f"tcp://127.0.0.1:{_free_port()}")
    try:
        router_w = torch.zeros(8, 128)
        with pytest.raises(ValueError):
            ep.ExpertParallelMoE(_Bank(4), _Bank(4), _Bank(4), router_w, top_k=2, ops=_Ops())
        layer = ep.ExpertParallelMoE(_Bank(8), _Bank(8), _Bank(8), router_w, top_k=2, max_tokens=4, ops=_Ops())
        with pytest.raises(ValueError):
            layer.forward(torch.zeros(5, 128, dtype=torch.bfloat16))
    finally:
        dist.destroy_process_group()


def test_bench_expert_parallel_leg_runs_on_cpu(monkeypatch):
    """bench.py's one-rank expert-parallel leg, run over gloo with the oracle's steps (its GPU run uses NCCL and
    the library): it initialises and releases its group, times the calls and compares with the fused layer,
    here the same steps composed on one process, bit for bit."""
    import bench
    import oracle
    from problems import build
    from weight_only_bit_route_b200 import synthetic as syn

    wl = syn.WORKLOADS[0]
    P = build(0, "random", experts=list(range(wl.E)), shared=True)
    ops = RefOps(oracle, P, 0, wl.E)
    x = _from_bits(syn.gen_x(wl, seed=7, T=5))

    def fused(x_, layer_, ws_):
        T = x_.shape[0]
        ids, w = ops.route(x_)
        off, rs, sr = ops.group(torch.zeros(T, wl.k, dtype=torch.int32), 1)
        rows = rs.to(torch.int64)
        ys = ops.experts(x_.index_select(0, rows // wl.k), ids.view(-1)[rows], w.view(-1)[rows])
        return ops.combine(ys, sr, T, ops.shared_expert(x_))

    class _Bank:
        E = wl.E

    layer = type("L", (), {"gate": _Bank(), "up": _Bank(), "down": _Bank(), "router_w": torch.from_numpy(P.Wr),
                           "router_bias": None, "shared": None})()
    fake = type("M", (), {"workspace": staticmethod(lambda *a: None), "layer_decode": staticmethod(fused)})
    def one_ms_each(fn, steps, *a, **kw):
        out = []
        for _ in range(steps):
            fn()
            out.append(1.0)
        return out

    monkeypatch.setattr(bench, "time_calls", one_ms_each)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: None)
    wl5 = syn.Workload(wl.name, 5, wl.H, wl.E, wl.F, wl.k, wl.fmt, True, wl.router_std, False)
    res = bench.measure_ep_one_rank(fake, wl5, x, layer, 2, None, None, None, backend="gloo", ops=ops)
    assert res["exact_vs_fused_layer"] is True
    assert res["world"] == 1 and res["tokens_per_s"] > 0
    import torch.distributed as dist
    assert not dist.is_initialized()
