"""The largest CSF case and the concurrency case, collected after the other GPU tests so that one of them
failing under `-x` cannot keep the rest from running.

- The compressed scale format at the size the benchmark expands: all 352 experts of one projection at the pages'
  shapes ("Step-5-Preview-NVFP4-Local", Format and Size), against the oracle's planes and the input bytes.
- Layer calls from two host threads at once, each on its own stream and workspace: bit-identical to one thread.
- Recording a layer as a graph launches nothing, so it adds nothing to the library's launch count.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_bit_route_b200 import moe

from problems import build, dev, dev_bf16, device_layer

pytestmark = pytest.mark.gpu


def _u32(t):
    return t.cpu().numpy().view(np.uint32)


def _ws(T, wl):
    return moe.workspace(T, wl.H, wl.E, wl.F, wl.k)


@pytest.mark.parametrize("R,C", [(1536, 256), (4096, 96)], ids=["gate_up_shape", "down_shape"])
def test_csf_full_layer_bitexact(R, C):
    """All 352 experts of one projection at the pages' shapes (the size the benchmark expands): each row's bytes
    sit in a 16-value window above a row base, with about 1 % replaced by arbitrary bytes (exceptions).  The
    encoder's planes equal the oracle's, the expansion of all experts returns the input, and the expansion of
    the routed experts writes exactly those."""
    rng = np.random.default_rng(13)
    E = 352
    base = rng.integers(0x30, 0x60, size=(E, R, 1), dtype=np.uint8)
    sc = (base + rng.integers(0, 16, size=(E, R, C), dtype=np.uint8)).astype(np.uint8)
    hit = rng.integers(0, 100, size=(E, R, C), dtype=np.uint8) == 0      # about 1 % of the bytes
    sc[hit] = rng.integers(0, 256, size=int(hit.sum()), dtype=np.uint8)
    f_ref, e_ref, s_ref = oracle.csf_encode(sc)
    f, e, s = moe.csf_encode(dev(sc))
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(f.cpu().numpy(), f_ref)
    assert np.array_equal(_u32(e), e_ref)
    out = moe.csf_decode(f, e, s, R, C)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), sc)
    counts = np.zeros(E, np.int32)
    counts[rng.choice(E, 60, replace=False)] = 1                    # a decode step's ~60 routed experts
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    part = torch.zeros(E, R, C, dtype=torch.uint8, device="cuda")
    moe.csf_decode(f, e, s, R, C, expert_offsets=dev(offsets), out=part)
    torch.cuda.synchronize()
    got = part.cpu().numpy()
    live = counts > 0
    assert np.array_equal(got[live], sc[live])
    assert not got[~live].any()


def test_layer_decode_from_two_host_threads():
    """Two host threads call moe_layer_decode at the same time, each on its own stream and workspace (the
    library releases the interpreter lock during a call; the shared expert's side stream is one per device,
    taken under a lock from its fork to its join): every call reproduces the one-thread result bit for bit."""
    import threading
    P = build(1, "random")
    L = device_layer(moe, P)
    x = dev_bf16(P.x)
    ref = moe.layer_decode(x, L, _ws(P.T, P.wl)).clone()
    torch.cuda.synchronize()
    outs, errors = [[], []], []

    def worker(i):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                ws = _ws(P.T, P.wl)
                for _ in range(20):
                    outs[i].append(moe.layer_decode(x, L, ws))
                if moe.read_status(ws) != 0:
                    errors.append(f"thread {i}: device status set")
            s.synchronize()
        except Exception as e:          # reported below, in the test's own thread
            errors.append(f"thread {i}: {e!r}")

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not any(t.is_alive() for t in threads), "a layer call did not return"
    assert not errors, errors
    torch.cuda.synchronize()
    for i in range(2):
        assert len(outs[i]) == 20
        bad = [j for j, y in enumerate(outs[i]) if not torch.equal(y, ref)]
        assert not bad, f"thread {i}: calls {bad} differ from the one-thread result"


def test_graph_recording_adds_no_launches():
    """moe_layer_graph_create records the layer's launches without running them: the launch count is the same
    before and after it, and one replay adds the recorded kernels (nine for the decode layer with a shared
    expert)."""
    P = build(1, "random")
    L = device_layer(moe, P)
    x = dev_bf16(P.x)
    ws = _ws(P.T, P.wl)
    torch.cuda.synchronize()
    n_rec = moe.launch_count()
    g = moe.LayerGraph(x, L, ws)
    assert moe.launch_count() == n_rec
    g.launch()
    torch.cuda.synchronize()
    assert moe.launch_count() - n_rec == 9
    assert moe.read_status(ws) == 0
    g.close()
